"""Throughput of the RWKV-4 WKV forward on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload NAME] [--variant auto|seq|scan|scan_ldg|step]

A step is one wkv4_forward call (the whole hot path: load, chunk summaries,
segment chaining, outputs, final state) over one batch of the workload,
default ``long_t65536`` (B=1, T=65536, C=2048, fp32 k/v/y, 0.1% of k spiked to
+30, fp32 state out: the largest single-GPU workload, 1.6 GB a call).  Inputs
are seeded synthetic data (rwkv_wkv_linear_b200.synth) resident in HBM; the
timed steps rotate over enough input sets that their total exceeds 3x the L2
cache, so no step reads another step's data from L2.  The K steps run as
CUDA-graph replays of the public call, right after about 0.25 s of untimed
replays (so the timed region starts on a busy GPU, not one waking from idle);
the device time of the region (CUDA events on the launching stream) is
max-reduced over ranks.

Under torchrun each rank processes its own batch (independent sequences, no
collective on the data path): weak scaling.

A decode workload (T = 1, e.g. ``--workload decode_b256``: B=256, C=5120,
bf16, 1024 calls) times the batched decode instead: one step is the whole
loop of wkv4_decode_step calls over one fp32 state updated in place, captured
as one CUDA graph; each call's k, v come from a pool of seeded inputs that
rotates over more than 3x the L2 cache.  The state (12 B a channel) stays
L2-resident across calls by design, so the line's GB/s is effective.
``--workload decode_slots_b256`` is the slot-indexed decode: each call serves
256 rows from a pool of 1024 states (wkv4_decode_step_slots), its slot ids
drawn per call.
``--workload token_shift_14b`` times the token shift feeding k, v and r
(wkv4_token_shift: B=4, T=1024, C=5120, bf16, three outputs); a step is one
call, the metric counts B*T*C elements as channel-steps.

``e2e`` is the same metric end to end from host memory: for the prefill
workloads one wkv4_forward_host call a step (pinned host buffers in, y and
the state out, the copies in both directions overlapped with the kernels in
chunks of T); for the decode and token-shift workloads the step's inputs are
copied in from pinned host memory, the call made and its outputs copied out,
on one stream.

``--impl reference`` times the fp64 CPU oracle on the same workload instead
(rank 0 only; other ranks exit).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "WKV-4 forward G channel-steps/s (B·T·C/s) and achieved HBM GB/s vs peak"
UNIT = "G channel-steps/s"
L2_BYTES = 126 * 1024 * 1024
VARIANTS = {"auto": 0, "seq": 1, "scan": 2, "scan_ldg": 3, "step": 4}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 20000 calls; 20 loops for a decode workload)")
    ap.add_argument("--warmup", type=int, default=None,
                    help="untimed steps (default 200 calls; 3 loops for a decode workload)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="long_t65536")
    ap.add_argument("--variant", default="auto", choices=sorted(VARIANTS))
    ap.add_argument("--graph-steps", type=int, default=500,
                    help="forward calls captured per CUDA graph")
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="run the workload's shape with this T instead (small profiling captures; "
                         "the line then names the shape it ran)")
    return ap.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """SM clock and throttle reasons sampled while the GPU works: NVML every
    few milliseconds from a thread of this process (reads only), else
    nvidia-smi every 50 ms.  summary(t0, t1) keeps the samples taken between
    host times t0 and t1 (the timed region), or, when the region is shorter
    than the sampling period, the last samples before t1."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu: str, period_s: float = 0.002):
        self.gpu = gpu
        self.period = period_s
        self.rows = []  # (host time, sm MHz, max MHz, set of reasons)
        self.proc = None
        self.t = None
        self.stop_flag = threading.Event()
        self.source = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = (pynvml.nvmlDeviceGetHandleByUUID(self.gpu.encode()) if self.gpu.startswith("GPU-")
                 else pynvml.nvmlDeviceGetHandleByIndex(int(self.gpu)))
            bits = {"hw_slowdown": pynvml.nvmlClocksThrottleReasonHwSlowdown,
                    "hw_thermal_slowdown": pynvml.nvmlClocksThrottleReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": pynvml.nvmlClocksThrottleReasonSwThermalSlowdown,
                    "sw_power_cap": pynvml.nvmlClocksThrottleReasonSwPowerCap}
            mx = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))

            def poll():
                while not self.stop_flag.is_set():
                    try:
                        sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                        r = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                        self.rows.append((time.perf_counter(), sm, mx,
                                          {n for n, b in bits.items() if r & b}))
                    except Exception:
                        pass
                    time.sleep(self.period)

            self.t = threading.Thread(target=poll, daemon=True)
            self.t.start()
            self.source = f"nvml every {self.period * 1e3:.0f} ms"
            return
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.source = "nvidia-smi every 50 ms"
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                try:
                    reasons = {n for n, val in zip(self.NAMES, parts[5:9])
                               if val.lower().startswith("active")}
                    self.rows.append((time.perf_counter(), float(parts[1]), float(parts[2]), reasons))
                except ValueError:
                    pass

    def stop(self):
        self.stop_flag.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.t is not None:
            self.t.join(timeout=5)

    def summary(self, t0=None, t1=None):
        rows = list(self.rows)
        window = "timed region"
        if t0 is not None and t1 is not None:
            inside = [r for r in rows if t0 <= r[0] <= t1]
            if len(inside) < 3:
                inside = [r for r in rows if r[0] <= t1][-5:]
                window = "last samples up to the end of the timed region (region shorter than the period)"
            rows = inside
        sm = [r[1] for r in rows]
        reasons = set()
        for r in rows:
            reasons |= r[3]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": rows[-1][2] if rows else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": self.source,
                "window": window}


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def io_bytes(wl):
    es = {"f32": 4, "f16": 2, "bf16": 2}[wl.dtype]
    return wl.B * wl.T * wl.C * es


def algorithmic_bytes(wl):
    """k, v (and r, gated) read + y written (I/O dtype) + state in (when given)
    and out (fp32 triples) + w, u (fp32)."""
    state = 12 * wl.B * wl.C
    return ((4 if wl.gated else 3) * io_bytes(wl) + (state if wl.random_state else 0) + state
            + 8 * wl.C)


def _code_only(text: str) -> str:
    """C/C++/CUDA source without its comments and blank lines (string and
    character literals kept), so that the hash below changes with the code only."""
    import re
    token = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\\n])*"|\'(?:\\.|[^\'\\\n])*\'', re.S)
    out = token.sub(lambda m: "" if m.group(0)[0] == "/" else m.group(0), text)
    return "\n".join(line.rstrip() for line in out.splitlines() if line.strip())


# host code that launches nothing of its own: the host-buffer pipeline only
# chains the forward's calls, so it does not change a kernel's traffic
_NOT_KERNEL_SOURCES = {"wkv4_host.cpp"}


def kernel_source_hash(csrc=None):
    """Hash of the kernel sources' code (comments and blank lines left out):
    the kernels, their launchers and the kernel choice.  A recorded
    DRAM-traffic figure applies only while it matches."""
    import hashlib
    h = hashlib.sha256()
    csrc = csrc or os.path.join(ROOT, "rwkv_wkv_linear_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name in _NOT_KERNEL_SOURCES:
            continue
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload, variant):
    """DRAM bytes per launch from the committed ncu summary (profiles/traffic.txt),
    or None when the kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        with open(path) as f:
            for line in f:
                parts = line.split()
                if not parts or parts[0].startswith("#") or parts[0] != f"{workload}/{variant}":
                    continue
                kv = dict(p.split("=", 1) for p in parts[1:] if "=" in p)
                if kv.get("kernel_source_hash") == kernel_source_hash():
                    return float(kv["dram_bytes_per_launch"])
    except OSError:
        pass
    return None


def cpu_baseline(wl, x):
    import oracle
    cores = len(os.sched_getaffinity(0))
    oracle.forward(x["k"][:1, :8], x["v"][:1, :8], x["w"], x["u"], None, nthreads=cores)
    r = None
    if wl.gated:
        from rwkv_wkv_linear_b200 import synth
        r = synth.receptance(wl)
    reps, t0 = 0, time.perf_counter()
    while True:
        if r is None:
            oracle.forward(x["k"], x["v"], x["w"], x["u"], x["state_in"], nthreads=cores)
        else:
            oracle.forward_gated(x["k"], x["v"], r, x["w"], x["u"], x["state_in"], nthreads=cores)
        reps += 1
        dt = time.perf_counter() - t0
        if reps >= 3 and dt > 1.0 or dt > 20.0:
            break
    value = wl.channel_steps * reps / dt / 1e9
    # one core, on the first channels of the workload (about 2 s of work)
    BC = wl.B * wl.C
    n_ch = max(1, min(BC, int(2.0 * value * 1e9 / max(1, cores) / wl.T)))
    smp = _ref_sample(x, wl, n_ch)
    t0 = time.perf_counter()
    oracle.forward(*smp, nthreads=1)
    value_1core = n_ch * wl.T / (time.perf_counter() - t0) / 1e9
    return {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"the whole workload ({wl.B}x{wl.T}x{wl.C}) x {reps} passes, fp64 C "
                      f"recurrence, {cores} threads over channels",
            "value_1core": value_1core,
            "sample_1core": f"{n_ch} of {BC} channels x all {wl.T} steps, one thread"}


def start_clocks(dev, local):
    import torch
    props = torch.cuda.get_device_properties(dev)
    uuid = getattr(props, "uuid", None)
    clocks = ClockSampler(f"GPU-{uuid}" if uuid is not None else str(local))
    clocks.start()
    return clocks


def busy_warmup(stream, graph, seconds: float = 0.25):
    """Untimed replays for about `seconds`, ending right before the timed
    region: its first steps then run at the clocks of a busy GPU."""
    import torch
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):
        while time.perf_counter() - t0 < seconds:
            graph.replay()
            stream.synchronize()


def host_call_us(wl, ks, vs, w, u, sis, ys, sos, variant, stream, rs=None,
                 calls: int = 200) -> float:
    """Host time of one wkv4_forward_variant call through the C ABI with its
    arguments already marshalled (argument checks, launch shape, tensor maps,
    launch): the cost an eager caller pays per call on top of the kernel."""
    import ctypes

    import torch
    from rwkv_wkv_linear_b200 import wkv4
    lib = wkv4.load()
    dt = {"f32": wkv4.F32, "f16": wkv4.F16, "bf16": wkv4.BF16}[wl.dtype]
    sp = ctypes.c_void_p(stream.cuda_stream)
    gated = rs is not None and rs[0] is not None
    fn = lib.wkv4_forward_gated_variant if gated else lib.wkv4_forward_variant
    args = [(wl.B, wl.T, wl.C, w.data_ptr(), u.data_ptr(), ks[j].data_ptr(), vs[j].data_ptr())
            + ((rs[j].data_ptr(),) if gated else ())
            + (sis[j].data_ptr() if sis[j] is not None else None, ys[j].data_ptr(),
               sos[j].data_ptr(), sp, dt, variant) for j in range(len(ks))]
    for a in args:  # first calls of each set (tensor maps encoded once)
        fn(*a)
    torch.cuda.synchronize()
    best = None
    for _ in range(3):
        t0 = time.perf_counter()
        for i in range(calls):
            rc = fn(*args[i % len(args)])
        t1 = time.perf_counter()
        torch.cuda.synchronize()
        if rc != 0:
            raise RuntimeError(f"wkv4_forward_variant failed ({rc})")
        us = (t1 - t0) / calls * 1e6
        best = us if best is None else min(best, us)
    return best


def max_over_ranks(ms: float, device=None) -> float:
    """The slowest rank's time (every rank takes part; a no-op for one process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(ms)
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(channel_steps_per_rank: int, steps: int, world: int, ms: float) -> float:
    """Whole-job G channel-steps/s: every rank processes its own batch (weak
    scaling) and the job takes as long as its slowest rank."""
    return world * channel_steps_per_rank * steps / (ms / 1e3) / 1e9


def run_native(args):
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from rwkv_wkv_linear_b200 import synth, wkv4

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wkv4.load()
    variant = VARIANTS[args.variant]
    wl = synth.workload(args.workload, **({"T": args.seq_len} if args.seq_len else {}))
    x = synth.forward_inputs(wl.replace(seed=wl.seed + 1000 * rank) if rank else wl)

    per_set = (3 if wl.gated else 2) * io_bytes(wl) + io_bytes(wl) + 24 * wl.B * wl.C
    nsets = max(2, -(-3 * L2_BYTES // per_set))
    nsets = min(nsets, max(2, int(20e9 // per_set)))
    w, u = x["w"].to(dev), x["u"].to(dev)
    ks = [x["k"].to(dev) for _ in range(nsets)]
    rs = [synth.receptance(wl).to(dev) for _ in range(nsets)] if wl.gated else [None] * nsets
    vs = [x["v"].to(dev) for _ in range(nsets)]
    sis = [x["state_in"].to(dev) if x["state_in"] is not None else None for _ in range(nsets)]
    ys = [torch.empty_like(ks[0]) for _ in range(nsets)]
    sos = [torch.empty((3, wl.B, wl.C), dtype=torch.float32, device=dev) for _ in range(nsets)]
    stream = torch.cuda.Stream(device=dev)

    def step(i):
        j = i % nsets
        if wl.gated:
            wkv4.forward_gated(ks[j], vs[j], rs[j], w, u, sis[j], y=ys[j], state_out=sos[j],
                               variant=variant, stream=stream)
        else:
            wkv4.forward(ks[j], vs[j], w, u, sis[j], y=ys[j], state_out=sos[j], variant=variant,
                         stream=stream)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    stream.synchronize()

    K = args.steps
    gsteps = max(1, min(args.graph_steps, K))
    graphs = []

    def capture(n, offset):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                step(offset + i)
        return g

    main_graph = capture(gsteps, 0)
    nrep, rem = divmod(K, gsteps)
    rem_graph = capture(rem, 0) if rem else None
    with torch.cuda.stream(stream):  # upload the graphs (untimed)
        main_graph.replay()
        if rem_graph is not None:
            rem_graph.replay()
    stream.synchronize()

    clocks = start_clocks(dev, local)
    busy_warmup(stream, main_graph)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_region0 = time.perf_counter()
    start.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(nrep):
            main_graph.replay()
        if rem_graph is not None:
            rem_graph.replay()
    end.record(stream)
    torch.cuda.synchronize()
    t_region1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    clocks.stop()
    ms = max_over_ranks(start.elapsed_time(end), dev)
    if wkv4.device_error() != 0:
        raise RuntimeError("device-side wait ran out during the timed region")
    host_us = host_call_us(wl, ks, vs, w, u, sis, ys, sos, variant, stream, rs)

    # end to end through the C ABI from pinned host buffers
    e2e = None
    if not args.no_e2e:
        kh, vh = x["k"].pin_memory(), x["v"].pin_memory()
        sih = x["state_in"].pin_memory() if x["state_in"] is not None else None
        yh = torch.empty_like(kh).pin_memory()
        soh = torch.empty((3, wl.B, wl.C), dtype=torch.float32).pin_memory()
        rh = synth.receptance(wl).pin_memory() if wl.gated else None
        # one wkv4_forward_host call a step: the host buffers go in and come
        # back in chunks of T, the copies overlapped with the kernels
        ws = torch.empty(wkv4.host_workspace_bytes(wl.B, wl.T, wl.C, kh.dtype, wl.gated),
                         dtype=torch.uint8, device=dev)

        def e2e_step():
            wkv4.forward_host(kh, vh, w, u, sih, r=rh, y=yh, state_out=soh, workspace=ws,
                              stream=stream)

        with torch.cuda.stream(stream):
            for _ in range(3):
                e2e_step()
        torch.cuda.synchronize()
        h2d = (3 if wl.gated else 2) * io_bytes(wl) + (12 * wl.B * wl.C if sih is not None else 0)
        d2h = io_bytes(wl) + 12 * wl.B * wl.C
        # about 4 GB of copies at most (three steps at the least)
        n_e2e = max(3, min(args.e2e_steps, int(4e9 // (h2d + d2h))))
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(n_e2e):
                e2e_step()
        e2.record(stream)
        torch.cuda.synchronize()
        t2_ms = max_over_ranks(s2.elapsed_time(e2), dev)
        e2e = {"value": job_throughput(wl.channel_steps, n_e2e, world, t2_ms),
               "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": n_e2e,
               "path": "wkv4_forward_host from pinned host buffers (copies in both directions "
                       "overlapped with the kernels, chunks of T chained through the state)"}

    if rank == 0:
        peak, peak_kind = measured_peaks()
        per_launch_s = ms / 1e3 / K
        achieved = algorithmic_bytes(wl) / per_launch_s / 1e9
        line = {
            "metric": METRIC,
            "value": job_throughput(wl.channel_steps, K, world, ms),
            "unit": UNIT,
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": ms / K,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "C": wl.C,
                       "io_dtype": wl.dtype, "state_in": "random" if wl.random_state else "none",
                       "gate": "y = sigmoid(r) wkv, r ~ N(0, 4)" if wl.gated else "none",
                       "global_batch": wl.B * world, "seq_len": wl.T,
                       "parallelism": f"independent sequences per rank (x{world})",
                       "kernel": args.variant,
                       "l2": f"inputs rotate over {nsets} sets ({nsets * per_set / 1e6:.0f} MB "
                             f"> 3x L2)",
                       "launch": f"CUDA graphs of {gsteps} calls, {nrep}+{1 if rem else 0} "
                                 "replays (one untimed upload replay each)",
                       "untimed": f"{args.warmup} warm-up calls before capture; about 0.25 s of "
                                  "replays right before the timed region"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": peak_kind,
                         "bytes_per_launch": algorithmic_bytes(wl),
                         "traffic": recorded_traffic(wl.name, args.variant)},
            "gpu_launches": K,
            "clocks": clocks.summary(t_region0, t_region1),
            "e2e": e2e,
            "host_us_per_call": host_us,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, x)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """The fp64 CPU oracle timed on this host's cores, on a bounded sample of
    the workload per step (all T steps of the first channels of the batch), so
    that --warmup W --steps K ends within a few minutes."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    from rwkv_wkv_linear_b200 import synth

    wl = synth.workload(args.workload)
    config = {"workload": wl.name, "B": wl.B, "T": wl.T, "C": wl.C, "io_dtype": wl.dtype}
    if wl.op == "token_shift":
        x = synth.shift_inputs(wl)
        for _ in range(args.warmup):
            cpu_baseline_shift(wl, x)
        t0 = time.perf_counter()
        base = None
        for _ in range(args.steps):
            base = cpu_baseline_shift(wl, x)
        dt = time.perf_counter() - t0
        line = {
            "impl": "reference", "metric": METRIC, "value": base["value"], "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "cpu_baseline": base,
            "e2e": {"value": base["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return
    if wl.slots:
        # the oracle's slot-indexed decode over a bounded sample of the calls
        for _ in range(args.warmup):
            cpu_baseline_slots(wl)
        t0 = time.perf_counter()
        base = None
        for _ in range(args.steps):
            base = cpu_baseline_slots(wl)
        dt = time.perf_counter() - t0
        config.update(calls=wl.steps, slots=wl.slots)
        line = {
            "impl": "reference", "metric": METRIC, "value": base["value"], "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "cpu_baseline": base,
            "e2e": {"value": base["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return
    if wl.T == 1:
        # a decode loop over one state is a forward over the calls' time axis
        wl, x = _decode_as_forward(wl)
        config.update(calls=synth.workload(args.workload).steps,
                      sampled_as=f"forward B={wl.B}, T={wl.T} (batch rows x calls)")
    else:
        x = synth.forward_inputs(wl)
    cores = len(os.sched_getaffinity(0))
    BC = wl.B * wl.C
    # calibrate: channel-steps per second of the oracle on this host
    n_cal = min(BC, max(1, 2_000_000 // wl.T))
    cal = _ref_sample(x, wl, n_cal)
    t0 = time.perf_counter()
    oracle.forward(*cal, nthreads=cores)
    rate = n_cal * wl.T / max(time.perf_counter() - t0, 1e-6)
    budget_s = 150.0 / max(1, args.steps + args.warmup)
    n_ch = int(min(BC, max(1, budget_s * rate / wl.T)))
    smp = _ref_sample(x, wl, n_ch)
    for _ in range(args.warmup):
        oracle.forward(*smp, nthreads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward(*smp, nthreads=cores)
    dt = time.perf_counter() - t0
    value = n_ch * wl.T * args.steps / dt / 1e9
    sample = (f"{n_ch} of {BC} channels x all {wl.T} steps per step (fp64 C recurrence, "
              f"{cores} threads)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _ref_sample(x, wl, n_ch):
    """The first n_ch flat channels (b*C + c) of the workload as one batch row:
    (k, v, w, u, state_in) fp64 arrays for oracle.forward."""
    import numpy as np
    BC = wl.B * wl.C
    ch = np.arange(n_ch)
    c = ch % wl.C
    k = x["k"].double().numpy().transpose(1, 0, 2).reshape(wl.T, BC)[:, :n_ch]
    v = x["v"].double().numpy().transpose(1, 0, 2).reshape(wl.T, BC)[:, :n_ch]
    w = x["w"].double().numpy()[c]
    u = x["u"].double().numpy()[c]
    s = None
    if x["state_in"] is not None:
        s = np.ascontiguousarray(x["state_in"].double().numpy().reshape(3, BC)[:, None, :n_ch])
    return (np.ascontiguousarray(k[None]), np.ascontiguousarray(v[None]), w, u, s)


def run_decode(args):
    """Batched decode: K loops of wl.steps wkv4_decode_step calls (one CUDA
    graph per loop) over one state; the device time of the K loops."""
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from rwkv_wkv_linear_b200 import synth, wkv4

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wkv4.load()
    wl = synth.workload(args.workload)
    if rank:
        wl = wl.replace(seed=wl.seed + 1000 * rank)
    w, u = (t.to(dev) for t in synth.decode_params(wl))
    call_io = 2 * io_bytes(wl)  # k, v of one call
    pool = max(8, -(-3 * L2_BYTES // call_io))
    ks, vs = [], []
    for s_ in range(pool):
        k, v = synth.decode_step_inputs(wl, s_)
        ks.append(k.to(dev))
        vs.append(v.to(dev))
    ys = [torch.empty_like(ks[0]) for _ in range(pool)]
    slots = wl.slots > 0
    state = synth.zero_state(wl.slots if slots else wl.B, wl.C).to(dev)
    ids = [synth.decode_slot_ids(wl, s_).to(dev) for s_ in range(pool)] if slots else None
    stream = torch.cuda.Stream(device=dev)
    n = wl.steps

    def call(kd, vd, yd, j):
        if slots:
            wkv4.decode_step_slots(kd, vd, w, u, state, ids[j], y=yd, stream=stream)
        else:
            wkv4.decode_step(kd, vd, w, u, state, y=yd, stream=stream)

    def loop():
        for s_ in range(n):
            j = s_ % pool
            call(ks[j], vs[j], ys[j], j)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            loop()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        loop()
    with torch.cuda.stream(stream):
        g.replay()  # upload (untimed)
    stream.synchronize()

    K = args.steps
    clocks = start_clocks(dev, local)
    busy_warmup(stream, g)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_region0 = time.perf_counter()
    start.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(K):
            g.replay()
    end.record(stream)
    torch.cuda.synchronize()
    t_region1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    clocks.stop()
    ms = max_over_ranks(start.elapsed_time(end), dev)
    if wkv4.device_error() != 0:
        raise RuntimeError("device-side error during the timed region")

    # end to end through the C ABI: every call's k, v (and slot ids) from
    # pinned host memory, its y back to the host
    e2e = None
    if not args.no_e2e:
        n_e2e = max(1, args.e2e_steps)
        kh = [ks[j % pool].cpu().pin_memory() for j in range(min(pool, n_e2e))]
        vh = [vs[j % pool].cpu().pin_memory() for j in range(min(pool, n_e2e))]
        ih = [ids[j % pool].cpu().pin_memory() for j in range(min(pool, n_e2e))] if slots else None
        yh = torch.empty_like(kh[0]).pin_memory()
        kd, vd, yd = ks[0], vs[0], ys[0]
        idd = torch.empty_like(ids[0]) if slots else None

        def e2e_call(j):
            kd.copy_(kh[j % len(kh)], non_blocking=True)
            vd.copy_(vh[j % len(vh)], non_blocking=True)
            if slots:
                idd.copy_(ih[j % len(ih)], non_blocking=True)
                wkv4.decode_step_slots(kd, vd, w, u, state, idd, y=yd, stream=stream)
            else:
                wkv4.decode_step(kd, vd, w, u, state, y=yd, stream=stream)
            yh.copy_(yd, non_blocking=True)

        with torch.cuda.stream(stream):
            for j in range(3):
                e2e_call(j)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        with torch.cuda.stream(stream):
            for j in range(n_e2e):
                e2e_call(j)
        e2.record(stream)
        torch.cuda.synchronize()
        t2_ms = max_over_ranks(s2.elapsed_time(e2), dev)
        e2e = {"value": job_throughput(wl.B * wl.C, n_e2e, world, t2_ms), "unit": UNIT,
               "h2d_bytes_per_step": call_io + (4 * wl.B if slots else 0),
               "d2h_bytes_per_step": io_bytes(wl),
               "steps": n_e2e, "step": "one decode call"}

    if rank == 0:
        peak, peak_kind = measured_peaks()
        calls = K * n
        # k, v, y + state read and written (+ the slot ids)
        call_bytes = 3 * io_bytes(wl) + 24 * wl.B * wl.C + (4 * wl.B if slots else 0)
        achieved = call_bytes / (ms / 1e3 / calls) / 1e9
        line = {
            "metric": METRIC,
            "value": job_throughput(wl.channel_steps, K, world, ms),
            "unit": UNIT,
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": ms / K,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "C": wl.C, "calls": n,
                       "io_dtype": wl.dtype,
                       "state": (f"fp32 pool of {wl.slots} states, rows named by per-call slot ids, "
                                 "in place, zero at the start") if slots else
                                "fp32, in place, zero at the start",
                       "global_batch": wl.B * world, "seq_len": n,
                       "parallelism": f"independent sequences per rank (x{world})",
                       "step": f"one decode loop of {n} "
                               f"{'wkv4_decode_step_slots' if slots else 'wkv4_decode_step'} calls",
                       "l2": f"k, v rotate over {pool} seeded call inputs "
                             f"({pool * call_io / 1e6:.0f} MB > 3x L2); the state is L2-resident",
                       "launch": f"one CUDA graph of {n} calls per step, {K} replays"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": peak_kind,
                         "bytes_per_launch": call_bytes, "effective": True,
                         "traffic": recorded_traffic(wl.name, "auto")},
            "gpu_launches": calls,
            "clocks": clocks.summary(t_region0, t_region1),
            "e2e": e2e,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_slots(wl) if slots else cpu_baseline_decode(wl)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_shift(args):
    """Token shift: K calls of wkv4_token_shift (CUDA graphs) over inputs that
    rotate over more than 3x L2; device time, e2e, the oracle on the host."""
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from rwkv_wkv_linear_b200 import synth, wkv4

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wkv4.load()
    wl = synth.workload(args.workload, **({"T": args.seq_len} if args.seq_len else {}))
    x = synth.shift_inputs(wl.replace(seed=wl.seed + 1000 * rank) if rank else wl)
    row = io_bytes(wl) // wl.T  # one [B][C] row
    per_set = 4 * io_bytes(wl) + 2 * row  # x read, three outputs written; x_prev, x_last
    nsets = max(2, -(-3 * L2_BYTES // per_set))
    mk, mv, mr = (m.to(dev) for m in x["mix"])
    xs = [x["x"].to(dev) for _ in range(nsets)]
    xps = [x["x_prev"].to(dev) for _ in range(nsets)]
    xls = [torch.empty_like(xps[0]) for _ in range(nsets)]
    outs = [[torch.empty_like(xs[0]) for _ in range(3)] for _ in range(nsets)]
    stream = torch.cuda.Stream(device=dev)
    lib = wkv4.load()
    dt = {"f32": wkv4.F32, "f16": wkv4.F16, "bf16": wkv4.BF16}[wl.dtype]
    sptr = stream.cuda_stream

    def call(xd, xpd, o, xld):
        rc = lib.wkv4_token_shift(wl.B, wl.T, wl.C, xd.data_ptr(), xpd.data_ptr(), mk.data_ptr(),
                                  mv.data_ptr(), mr.data_ptr(), o[0].data_ptr(), o[1].data_ptr(),
                                  o[2].data_ptr(), xld.data_ptr(), sptr, dt)
        if rc != 0:
            raise RuntimeError(f"wkv4_token_shift failed ({rc})")

    def step(i):
        j = i % nsets
        call(xs[j], xps[j], outs[j], xls[j])

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    stream.synchronize()
    K = args.steps
    gsteps = max(1, min(args.graph_steps, K))
    nrep, rem = divmod(K, gsteps)
    graphs = []
    for n in [gsteps] + ([rem] if rem else []):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                step(i)
        graphs.append(g)
    with torch.cuda.stream(stream):
        for g in graphs:
            g.replay()  # upload (untimed)
    stream.synchronize()
    clocks = start_clocks(dev, local)
    busy_warmup(stream, graphs[0])
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_region0 = time.perf_counter()
    start.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(nrep):
            graphs[0].replay()
        if rem:
            graphs[1].replay()
    end.record(stream)
    torch.cuda.synchronize()
    t_region1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    clocks.stop()
    ms = max_over_ranks(start.elapsed_time(end), dev)

    e2e = None
    if not args.no_e2e:
        xh, xph = x["x"].pin_memory(), x["x_prev"].pin_memory()
        oh = [torch.empty_like(xh).pin_memory() for _ in range(3)]
        xlh = torch.empty_like(xph).pin_memory()

        def e2e_step():
            xs[0].copy_(xh, non_blocking=True)
            xps[0].copy_(xph, non_blocking=True)
            call(xs[0], xps[0], outs[0], xls[0])
            for o_h, o_d in zip(oh, outs[0]):
                o_h.copy_(o_d, non_blocking=True)
            xlh.copy_(xls[0], non_blocking=True)

        with torch.cuda.stream(stream):
            for _ in range(3):
                e2e_step()
        torch.cuda.synchronize()
        n_e2e = max(1, args.e2e_steps)
        if world > 1:
            dist.barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(n_e2e):
                e2e_step()
        e2.record(stream)
        torch.cuda.synchronize()
        t2_ms = max_over_ranks(s2.elapsed_time(e2), dev)
        e2e = {"value": job_throughput(wl.channel_steps, n_e2e, world, t2_ms), "unit": UNIT,
               "h2d_bytes_per_step": io_bytes(wl) + row,
               "d2h_bytes_per_step": 3 * io_bytes(wl) + row, "steps": n_e2e}

    if rank == 0:
        peak, peak_kind = measured_peaks()
        call_bytes = 4 * io_bytes(wl) + 2 * row + 12 * wl.C
        achieved = call_bytes / (ms / 1e3 / K) / 1e9
        line = {
            "metric": METRIC, "value": job_throughput(wl.channel_steps, K, world, ms),
            "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "C": wl.C, "io_dtype": wl.dtype,
                       "outputs": "xk, xv, xr and x_last", "global_batch": wl.B * world,
                       "seq_len": wl.T, "parallelism": f"independent sequences per rank (x{world})",
                       "l2": f"inputs rotate over {nsets} sets ({nsets * per_set / 1e6:.0f} MB > 3x L2)",
                       "launch": f"CUDA graphs of {gsteps} calls"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": peak_kind,
                         "bytes_per_launch": call_bytes,
                         "traffic": recorded_traffic(wl.name, "auto")},
            "gpu_launches": K, "clocks": clocks.summary(t_region0, t_region1), "e2e": e2e,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_shift(wl, x)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def cpu_baseline_shift(wl, x):
    """The oracle's token shift over the whole workload (numpy, one thread)."""
    import oracle
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.token_shift(x["x"], x["x_prev"], x["mix"])
        reps += 1
        dt = time.perf_counter() - t0
        if reps >= 3 and dt > 1.0 or dt > 20.0:
            break
    return {"value": wl.channel_steps * reps / dt / 1e9, "unit": UNIT, "cores": 1,
            "kind": "oracle",
            "sample": f"the whole workload ({wl.B}x{wl.T}x{wl.C}) x {reps} passes, fp64 numpy"}


def _decode_as_forward(wl, rows: int = 16, calls: int = 128):
    """The first `rows` batch rows and `calls` calls of a decode workload as
    forward inputs (B = rows, T = calls), with its w, u and the zero state."""
    import torch
    from rwkv_wkv_linear_b200 import synth
    w, u = synth.decode_params(wl)
    calls = min(calls, wl.steps)
    ks, vs = [], []
    for s_ in range(calls):
        k, v = synth.decode_step_inputs(wl, s_)
        ks.append(k[:rows])
        vs.append(v[:rows])
    x = {"w": w, "u": u, "k": torch.stack(ks, dim=1), "v": torch.stack(vs, dim=1),
         "state_in": None}
    return wl.replace(name=wl.name, B=min(rows, wl.B), T=calls, steps=1), x


def cpu_baseline_decode(wl):
    """The oracle over a bounded sample of the decode workload (see
    _decode_as_forward)."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    ws, x = _decode_as_forward(wl)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.forward(x["k"], x["v"], x["w"], x["u"], None, nthreads=cores)
        reps += 1
        dt = time.perf_counter() - t0
        if reps >= 3 and dt > 1.0 or dt > 20.0:
            break
    return {"value": ws.channel_steps * reps / dt / 1e9, "unit": UNIT, "cores": cores,
            "kind": "oracle",
            "sample": f"batch rows 0..{ws.B - 1} of {wl.B} x calls 0..{ws.T - 1} of {wl.steps}, "
                      f"C={wl.C} ({ws.channel_steps} channel-steps) x {reps} passes, fp64 C "
                      f"recurrence, {cores} threads over channels"}


def _slots_sample(wl, rows: int = 16, pool: int = 64, calls: int = 32):
    """A bounded sample of a slot-indexed decode workload for the oracle: the
    first `rows` rows of each of the first `calls` calls, their ids folded
    into a pool of `pool` states (ids mod pool, made distinct per call)."""
    import numpy as np
    from rwkv_wkv_linear_b200 import synth
    w, u = synth.decode_params(wl)
    calls = min(calls, wl.steps)
    steps = []
    for s_ in range(calls):
        k, v = synth.decode_step_inputs(wl, s_)
        ids = synth.decode_slot_ids(wl, s_).numpy()[:rows] % pool
        _, first = np.unique(ids, return_index=True)  # one row per slot within a call
        keep = np.sort(first)
        steps.append((k[:rows][keep], v[:rows][keep], ids[keep]))
    return w, u, steps, pool


def cpu_baseline_slots(wl):
    """The oracle's slot-indexed decode over a bounded sample (_slots_sample)."""
    import numpy as np
    import oracle
    cores = len(os.sched_getaffinity(0))
    w, u, steps, pool = _slots_sample(wl)
    n_ch = sum(len(ids) for _, _, ids in steps) * wl.C
    reps, t0 = 0, time.perf_counter()
    while True:
        st = oracle.empty_state(pool, wl.C)
        for k, v, ids in steps:
            _, st, _ = oracle.decode_slots(k, v, w, u, st, ids)
        reps += 1
        dt = time.perf_counter() - t0
        if reps >= 3 and dt > 1.0 or dt > 20.0:
            break
    return {"value": n_ch * reps / dt / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{len(steps)} calls x up to 16 rows of {wl.B} from a pool of {pool} states, "
                      f"C={wl.C} ({n_ch} channel-steps) x {reps} passes, fp64 C recurrence per row"}


def main():
    args = parse()
    from rwkv_wkv_linear_b200 import synth
    decode = synth.workload(args.workload).T == 1
    if args.steps is None:
        args.steps = 20 if decode else 20000
    if args.warmup is None:
        args.warmup = 3 if decode else 200
    if args.impl == "reference":
        run_reference(args)
    elif synth.workload(args.workload).op == "token_shift":
        run_shift(args)
    elif decode:
        run_decode(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
