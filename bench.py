"""Benchmark: RWKV-4 WKV forward + backward on the 1.5B-width training shape.

One step = one forward (y and state checkpoints) + one backward (gk, gv, gw,
gu) over B=8, T=4096, C=2048 fp32, keys with 1 % +-U(20,40) outliers,
gy ~ N(0,1), all synthetic and seeded.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torch.distributed.run, one process per GPU) every rank
runs its own independent problem (the operator shards over batch rows with no
exchange); ``value`` is the whole job's elements/s over the max of the ranks'
device times.  ``--impl reference`` times the fp64 CPU oracle on the host on a
bounded sample of the same workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

B, T, C = 8, 4096, 2048
SEED = 20261204  # seed base + workload index 2
ELEM = B * T * C
FWD_BYTES = 3 * 4 * ELEM                     # k, v read; y written
BWD_BYTES = 5 * 4 * ELEM + 2 * 4 * C         # k, v, gy read; gk, gv written; gw, gu
METRIC = "WKV fwd+bwd elements/s and HBM GB/s (% of peak) at B8·T4096·C2048"
WORKLOAD = "RWKV-4 WKV forward+backward, fp32, B=8 T=4096 C=2048, 1% +-U(20,40) key outliers"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _gpu_id(local):
    """The UUID of CUDA device ``local`` ("GPU-..."), which NVML and nvidia-smi
    accept whatever CUDA_VISIBLE_DEVICES renumbers; the index if unknown."""
    try:
        import torch

        u = torch.cuda.get_device_properties(local).uuid
        return "GPU-" + str(u)
    except Exception:
        return local


class ClockSampler:
    """Samples SM clocks and throttle reasons while the benchmark runs (read only).

    NVML (the driver's management library, through nvidia_ml_py) answers in
    microseconds, so even a timed region of a few milliseconds holds many
    samples; without it, nvidia-smi is polled one query at a time."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    # NVML clocks-event reason bits for the names above
    NVML_BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}

    def __init__(self, index, period: float = 0.05):
        self.index = _gpu_id(index)  # the device's UUID where torch reports one, else its index
        self.period = period
        self.samples = []  # (time, sm_mhz, max_mhz, [reasons])
        self._stop = threading.Event()
        self.window = None
        self.source = None

    def _poll_nvml(self):
        import pynvml

        pynvml.nvmlInit()
        try:
            h = (pynvml.nvmlDeviceGetHandleByUUID(self.index) if isinstance(self.index, str)
                 else pynvml.nvmlDeviceGetHandleByIndex(self.index))
            sm_max = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.source = "nvml"
            while not self._stop.is_set():
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                bits = get_reasons(h)
                reasons = [n for n, b in self.NVML_BITS.items() if bits & b]
                self.samples.append((time.perf_counter(), float(sm), float(sm_max), reasons))
                self._stop.wait(0.002)
        finally:
            pynvml.nvmlShutdown()

    def _poll_smi(self):
        self.source = "nvidia-smi"
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                     timeout=5).stdout.strip()
                parts = [x.strip() for x in out.split(",")]
                if len(parts) >= 8:
                    reasons = [n for n, v in zip(self.NAMES, parts[4:8]) if v.lower().startswith("active")]
                    self.samples.append((time.perf_counter(), float(parts[0]), float(parts[1]), reasons))
            except Exception:
                return
            self._stop.wait(self.period)

    def _poll(self):
        try:
            self._poll_nvml()
        except Exception:
            if not self.samples:
                self._poll_smi()

    def __enter__(self):
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()
        t_end = time.perf_counter() + 2.0  # the first sample before anything is timed
        while not self.samples and self.thread.is_alive() and time.perf_counter() < t_end:
            time.sleep(0.001)
        return self

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def __exit__(self, *a):
        self._stop.set()
        self.thread.join(timeout=10)

    def summary(self):
        if not self.samples:
            return None
        chosen, where = self.samples, "benchmark run (warm-up and timed steps)"
        if self.window is not None:
            t0, t1 = self.window
            inside = [x for x in self.samples if t0 <= x[0] <= t1]
            if inside:
                chosen, where = inside, "timed region"
        sm = sorted(x[1] for x in chosen)
        reasons = sorted({r for x in chosen for r in x[3]})
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": chosen[-1][2], "reasons": reasons,
                "samples": len(chosen), "window": where, "source": self.source}


# kernel name in profiles/traffic.json -> prefix of the source files it is built from
_TRAFFIC_SOURCES = {"wkv4_bwd_kernel": "wkv4_bwd", "wkv5_fwd_tc_kernel": "wkv5_fwd", "wkv4_step_kernel": "wkv4_step",
                    "wkv5_step_kernel": "wkv5_step", "wkv6_fwd_tc_kernel": "wkv6_fwd",
                    "wkv5_step_kernel/finch": "wkv5_step", "wkv4_bwd_kernel/gated": "wkv4_bwd",
                    "rwkv_wkv5_backward": ("wkv5_fwd", "wkv5_bwd"), "rwkv_wkv6_backward": "wkv6_bwd"}


def _kernel_source_hash(kernel="wkv4_bwd_kernel"):
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "rwkv_wkv_recurrence_b200", "csrc")
    prefixes = _TRAFFIC_SOURCES[kernel]
    units = {p + ".cu" for p in ((prefixes,) if isinstance(prefixes, str) else prefixes)}
    for f in sorted(os.listdir(csrc)):
        if f in units or f.endswith(".cuh") or f == "launch.h":
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()[:16]


def _recorded_traffic(kernel="wkv4_bwd_kernel"):
    """DRAM bytes per launch of `kernel` from the committed ncu capture, if it was
    taken on the kernel source as it is now (else None)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            d = json.load(f)[kernel]
        return d["dram_bytes_per_launch"] if d.get("source_hash") == _kernel_source_hash(kernel) else None
    except Exception:
        return None


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _oracle_sample(n_ch):
    """The bounded sample the oracle is timed on: all batch rows and steps of n_ch of the
    C channels (every C/n_ch-th), as fp64 [B, T, n_ch] arrays."""
    import numpy as np
    import torch

    import wkv_inputs as wi

    chans = torch.arange(0, C, C // n_ch)[:n_ch]
    w, u = wi.wkv4_params(SEED, C)
    b_sel = torch.arange(B).repeat_interleave(n_ch)
    c_sel = chans.repeat(B)

    def field(kind, out=False):
        x = wi.btc_field(kind, SEED, B, T, C, b_sel=b_sel, c_sel=c_sel, outliers=out)  # [T, B*n]
        return np.ascontiguousarray(x.T.reshape(B, n_ch, T).permute(0, 2, 1).double().numpy())

    return (w[chans].double().numpy(), u[chans].double().numpy(), field("k", True), field("v"), field("gy"),
            f"all {B} batch rows x {T} steps x {n_ch} of {C} channels (every {C // n_ch}th), fp64")


def _oracle_step(oracle, ws, us, k, v, gy):
    oracle.wkv4_forward(ws, us, k, v)
    oracle.wkv4_backward(ws, us, k, v, gy)


def run_reference(args):
    """The fp64 CPU oracle, as it stands, on a bounded sample of the workload."""
    world, rank, _ = _dist()
    if rank != 0:
        return
    import oracle

    ws, us, k, v, gy, sample = _oracle_sample(args.ref_channels)
    elems = B * T * args.ref_channels
    for _ in range(args.warmup):
        _oracle_step(oracle, ws, us, k, v, gy)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(oracle, ws, us, k, v, gy)
    dt = (time.perf_counter() - t0) / args.steps
    val = elems / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "elements/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "T": T, "C": C, "sample_channels": args.ref_channels},
        "cpu_baseline": {"value": val, "unit": "elements/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": val, "unit": "elements/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(seconds_target=10.0, n_ch=256):
    """Times the oracle (fp64, OpenMP) on the reference arm's sample (all batch rows and
    steps of n_ch channels), on all host cores and on one thread, about seconds_target
    in total."""
    import oracle

    ws, us, k, v, gy, sample = _oracle_sample(n_ch)
    all_cores = oracle.num_threads()

    def timed(budget):
        reps, t0 = 0, time.perf_counter()
        while True:
            _oracle_step(oracle, ws, us, k, v, gy)
            reps += 1
            if time.perf_counter() - t0 >= budget or reps >= 1000:
                return reps, (time.perf_counter() - t0) / reps

    _oracle_step(oracle, ws, us, k, v, gy)  # warm
    reps, dt = timed(0.5 * seconds_target)
    oracle.set_num_threads(1)
    try:
        reps1, dt1 = timed(0.5 * seconds_target)
    finally:
        oracle.set_num_threads(all_cores)
    elems = B * T * n_ch
    return {"value": elems / dt, "unit": "elements/s", "cores": all_cores, "kind": "oracle",
            "one_thread": {"value": elems / dt1, "unit": "elements/s", "cores": 1, "reps": reps1},
            "sample": f"{reps} x forward+backward over {sample}"}


class _Nvtx:
    """NVTX range around a library call (names the call in an nsys or ncu timeline)."""

    def __init__(self, name):
        self.name = name

    def __enter__(self):
        import torch

        torch.cuda.nvtx.range_push(self.name)

    def __exit__(self, *a):
        import torch

        torch.cuda.nvtx.range_pop()


def _stats(ms_list):
    """Mean, median and min of per-step device times (ms)."""
    xs = sorted(ms_list)
    n = len(xs)
    med = xs[n // 2] if n % 2 else 0.5 * (xs[n // 2 - 1] + xs[n // 2])
    return {"mean": sum(xs) / n, "median": med, "min": xs[0], "n": n}


def run_ours(args):
    import torch

    import rwkv_wkv_recurrence_b200 as rw
    import wkv_inputs as wi
    from rwkv_wkv_recurrence_b200.dist_timing import max_over_ranks, rank_seed, weak_scaling_throughput

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    h = rw.lib()
    stream = torch.cuda.current_stream()
    # each rank its own independent problem (weak scaling)
    p = wi.wkv4_problem(B, T, C, rank_seed(SEED, rank), outliers=True, with_gy=True, device=dev)
    w, u, k, v, gy = p["w"], p["u"], p["k"], p["v"], p["gy"]
    y = torch.empty_like(k)
    gk, gv = torch.empty_like(k), torch.empty_like(k)
    gw = torch.empty(C, device=dev)
    gu = torch.empty(C, device=dev)
    nck = int(h.rwkv_wkv4_num_checkpoints(T, rw.CHUNK_LEN))
    ck = torch.empty((nck, 3, B, C), device=dev)
    fws = int(h.rwkv_wkv4_forward_workspace_bytes(B, T, C, rw.ALGO_AUTO))
    bws = int(h.rwkv_wkv4_backward_workspace_bytes(B, T, C, rw.CHUNK_LEN, 1))
    fw = torch.empty(max(fws, 1), dtype=torch.uint8, device=dev)
    bw = torch.empty(bws, dtype=torch.uint8, device=dev)
    sp = rw._stream(stream)
    P = rw._ptr

    def fwd():
        with _Nvtx("rwkv_wkv4_forward"):
            s = h.rwkv_wkv4_forward(B, T, C, rw.F32, P(w), P(u), P(k), P(v), P(y), None, None, P(ck),
                                    rw.CHUNK_LEN, rw.ALGO_AUTO, P(fw), fws, sp)
        if s:
            raise rw.RwkvError("rwkv_wkv4_forward", s)

    def bwd():
        with _Nvtx("rwkv_wkv4_backward"):
            s = h.rwkv_wkv4_backward(B, T, C, rw.F32, P(w), P(u), P(k), P(v), P(gy), None, P(ck), rw.CHUNK_LEN,
                                     P(gk), P(gv), P(gw), P(gu), P(bw), bws, sp)
        if s:
            raise rw.RwkvError("rwkv_wkv4_backward", s)

    launches_per_step = 3  # forward scan; backward scan + gw/gu batch reduction

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        fwd()
        bwd()
    barrier()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        wall0 = time.perf_counter()
        start.record(stream)
        for i in range(args.steps):
            evs[i][0].record(stream)
            fwd()
            evs[i][1].record(stream)
            bwd()
            evs[i][2].record(stream)
        end.record(stream)
        barrier()
        clk.mark(wall0, time.perf_counter())
    rw.rwkv_check_device_error()
    total_ms = start.elapsed_time(end)
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    bwd_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    step_stats = _stats([e[0].elapsed_time(e[2]) for e in evs])
    ms_step = max_over_ranks(total_ms, dev) / args.steps
    value = weak_scaling_throughput(ELEM, world, ms_step)

    # end to end through the public API with host buffers (pinned), copies timed.  Each step copies its
    # inputs in and its results out; the results leave from one of two output sets while the next
    # step's inputs arrive (PCIe is full duplex) and the step after that computes into the other set.
    hk, hv, hgy = (x.cpu().pin_memory() for x in (k, v, gy))
    hw, hu = w.cpu().pin_memory(), u.cpu().pin_memory()
    hy, hgk, hgv = (torch.empty_like(hk).pin_memory() for _ in range(3))
    hgw, hgu = torch.empty(C).pin_memory(), torch.empty(C).pin_memory()
    outs = [(y, gk, gv, gw, gu), tuple(torch.empty_like(x) for x in (y, gk, gv, gw, gu))]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def e2e_run(n):
        ev = [dict(inp=torch.cuda.Event(), done=torch.cuda.Event(), out=torch.cuda.Event()) for _ in range(n)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(s_in)
        for i in range(n):
            yy, gkk, gvv, gww, guu = outs[i % 2]
            with torch.cuda.stream(s_in), _Nvtx("e2e h2d"):
                if i >= 1:
                    s_in.wait_event(ev[i - 1]["done"])  # the previous step has read k, v, gy
                for dst, src in ((k, hk), (v, hv), (gy, hgy), (w, hw), (u, hu)):
                    dst.copy_(src, non_blocking=True)
                ev[i]["inp"].record(s_in)
            stream.wait_event(ev[i]["inp"])
            if i >= 2:
                stream.wait_event(ev[i - 2]["out"])  # this output set has left
            with _Nvtx("rwkv_wkv4_forward"):
                st = h.rwkv_wkv4_forward(B, T, C, rw.F32, P(w), P(u), P(k), P(v), P(yy), None, None, P(ck),
                                         rw.CHUNK_LEN, rw.ALGO_AUTO, P(fw), fws, sp)
            if st:
                raise rw.RwkvError("rwkv_wkv4_forward", st)
            with _Nvtx("rwkv_wkv4_backward"):
                st = h.rwkv_wkv4_backward(B, T, C, rw.F32, P(w), P(u), P(k), P(v), P(gy), None, P(ck), rw.CHUNK_LEN,
                                          P(gkk), P(gvv), P(gww), P(guu), P(bw), bws, sp)
            if st:
                raise rw.RwkvError("rwkv_wkv4_backward", st)
            ev[i]["done"].record(stream)
            with torch.cuda.stream(s_out), _Nvtx("e2e d2h"):
                s_out.wait_event(ev[i]["done"])
                for dst, src in ((hy, yy), (hgk, gkk), (hgv, gvv), (hgw, gww), (hgu, guu)):
                    dst.copy_(src, non_blocking=True)
                ev[i]["out"].record(s_out)
        e1.record(s_out)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    e2e_steps = max(2, min(args.steps, 20))  # the first input copy and the last result copy are not overlapped
    e2e_run(2)  # warm-up
    barrier()
    e2e_val = weak_scaling_throughput(ELEM, world, max_over_ranks(e2e_run(e2e_steps), dev))
    barrier()

    if rank == 0:
        peak, peak_kind = _peaks()
        bwd_gbs = BWD_BYTES / (bwd_ms * 1e-3) / 1e9
        step_gbs = (FWD_BYTES + BWD_BYTES) / (ms_step * 1e-3) / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": "elements/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": B, "T": T, "C": C, "per_gpu_problem": "independent",
                       "l2": "no flush: every input (k, v, gy: 268 MB each) is larger than the 126 MB L2",
                       "parallelism": f"{world} independent problems, no collective"},
            "hbm_gbs_step": step_gbs, "hbm_frac_step": step_gbs / peak,
            "step_ms": step_stats,
            "kernels_ms": {"wkv4_forward": fwd_ms, "wkv4_backward": bwd_ms},
            "roofline": {"bound": "hbm", "kernel": "wkv4_bwd_kernel (+ its gw/gu batch reduction)",
                         "achieved": bwd_gbs, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": bwd_gbs / peak,
                         "traffic": args.traffic if args.traffic is not None else _recorded_traffic()},
            "e2e": {"value": e2e_val, "unit": "elements/s",
                    "h2d_bytes_per_step": 3 * 4 * ELEM + 2 * 4 * C, "d2h_bytes_per_step": 3 * 4 * ELEM + 2 * 4 * C},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(),
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def _timed(fn, steps, warmup, stream, local):
    """W untimed calls, then K calls bracketed by synchronisation, CUDA events
    on the launching stream; returns (mean ms per call, clock summary, per-call
    mean/median/min)."""
    import torch

    for _ in range(warmup):
        fn(0)
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        wall0 = time.perf_counter()
        evs[0].record(stream)
        for i in range(steps):
            fn(i)
            evs[i + 1].record(stream)
        torch.cuda.synchronize()
        clk.mark(wall0, time.perf_counter())
    stats = _stats([evs[i].elapsed_time(evs[i + 1]) for i in range(steps)])
    return evs[0].elapsed_time(evs[-1]) / steps, clk.summary(), stats


def run_decode(args):
    """Recurrent decode: 4096 independent streams x 4096 channels, one token per
    step for every stream (state in and out in place), inputs of 256 distinct
    tokens pre-generated on the device and cycled."""
    import torch

    import rwkv_wkv_recurrence_b200 as rw
    import wkv_inputs as wi

    _, _, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    Bd, Cd, Tp, Td = 4096, 4096, 128, 256
    seed = SEED + 1
    w, u = wi.wkv4_params(seed, Cd, device=dev)
    kp = wi.btc_field("k", seed, Bd, Tp + Td, Cd, t0=0, t1=Tp, device=dev)
    vp = wi.btc_field("v", seed, Bd, Tp + Td, Cd, t0=0, t1=Tp, device=dev)
    _, st = rw.rwkv_wkv4_forward(w, u, kp, vp, return_state=True)
    del kp, vp
    ks = [wi.btc_field("k", seed, Bd, Tp + Td, Cd, t0=t, t1=t + 1, device=dev)[:, 0].contiguous()
          for t in range(Tp, Tp + Td)]
    vs = [wi.btc_field("v", seed, Bd, Tp + Td, Cd, t0=t, t1=t + 1, device=dev)[:, 0].contiguous()
          for t in range(Tp, Tp + Td)]
    y = torch.empty(Bd, Cd, device=dev)
    h = rw.lib()
    stream = torch.cuda.current_stream()
    sp, P = rw._stream(stream), rw._ptr

    def step(i):
        j = i % Td
        s = h.rwkv_wkv4_step(Bd, Cd, rw.F32, P(w), P(u), P(ks[j]), P(vs[j]), P(y), P(st), P(st), sp)
        if s:
            raise rw.RwkvError("rwkv_wkv4_step", s)

    ms, clk, stats = _timed(step, args.steps, args.warmup, stream, local)
    rw.rwkv_check_device_error()
    graph = _graph_decode_timing(rw, h, st, w, u, ks, vs, y, Bd, Cd, Td, dev)
    lanes = Bd * Cd
    bytes_step = 36 * lanes  # state 12 B in + 12 B out, k, v, y 4 B each
    gbs = bytes_step / (ms * 1e-3) / 1e9
    peak, kind = _peaks()
    print(json.dumps({
        "metric": "WKV-4 decode lane-steps/s and HBM GB/s (4096 streams x C4096)", "value": lanes / (ms * 1e-3),
        "unit": "lane-steps/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "RWKV-4 WKV decode, fp32, 4096 streams x C=4096, state in place, 256 tokens cycled",
                   "l2": "no flush: 604 MB moved per step, above the 126 MB L2"},
        "roofline": {"bound": "hbm", "kernel": "wkv4_step_kernel", "achieved": gbs, "peak": peak,
                     "peak_kind": kind, "unit": "GB/s", "frac": gbs / peak,
                     "traffic": _recorded_traffic("wkv4_step_kernel")},
        "gpu_launches": args.steps, "clocks": clk, "call_ms": stats, "cuda_graph": graph}), flush=True)


def _graph_decode_timing(rw, h, st, w, u, ks, vs, y, Bd, Cd, Td, dev):
    """The decode loop as a CUDA graph: the Td-token loop of the full shape captured
    once and replayed, and the same for a small batch of 16 streams, where each
    step is a few microseconds and launch overhead matters; eager timing beside it."""
    import torch

    P = rw._ptr

    def loop(stream, nb, state, kk, vv, yy):
        sp = rw._stream(stream)
        for j in range(Td):
            s = h.rwkv_wkv4_step(nb, Cd, rw.F32, P(w), P(u), P(kk[j]), P(vv[j]), P(yy), P(state), P(state), sp)
            if s:
                raise rw.RwkvError("rwkv_wkv4_step", s)

    def time_it(fn, reps):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps / Td

    out = {"steps_per_graph": Td}
    for name, nb in (("full", Bd), ("16_streams", 16)):
        state = st[:, :nb].contiguous() if nb != Bd else st
        kk = ks if nb == Bd else [x[:nb].contiguous() for x in ks]
        vv = vs if nb == Bd else [x[:nb].contiguous() for x in vs]
        yy = y if nb == Bd else y[:nb].contiguous()
        eager_ms = time_it(lambda: loop(torch.cuda.current_stream(), nb, state, kk, vv, yy), 3)
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            loop(side, nb, state, kk, vv, yy)  # warm the launch path on the capture stream
        torch.cuda.current_stream().wait_stream(side)
        with torch.cuda.graph(g):
            loop(torch.cuda.current_stream(), nb, state, kk, vv, yy)
        graph_ms = time_it(g.replay, 3)
        out[name] = {"streams": nb, "eager_us_per_step": eager_ms * 1e3, "graph_us_per_step": graph_ms * 1e3}
        del g
    return out


def run_train_gated(args):
    """Receptance-gated RWKV-4 training step: o = sigmoid(r) * WKV forward and its
    backward (gk, gv, gr, gw, gu), fp32, B=8 T=4096 C=2048, as the headline step."""
    import torch

    import rwkv_wkv_recurrence_b200 as rw
    import wkv_inputs as wi

    _, _, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    p = wi.wkv4_problem(B, T, C, SEED, outliers=True, with_gy=True, gated=True, device=dev)
    w, u, k, v, r, go = p["w"], p["u"], p["k"], p["v"], p["r"], p["go"]
    o = torch.empty_like(k)
    gk, gv, gr = torch.empty_like(k), torch.empty_like(k), torch.empty_like(k)
    gw, gu = torch.empty(C, device=dev), torch.empty(C, device=dev)
    h = rw.lib()
    nck = int(h.rwkv_wkv4_num_checkpoints(T, rw.CHUNK_LEN))
    ck = torch.empty((nck, 3, B, C), device=dev)
    fws = int(h.rwkv_wkv4_forward_workspace_bytes(B, T, C, rw.ALGO_AUTO))
    bws = int(h.rwkv_wkv4_backward_workspace_bytes(B, T, C, rw.CHUNK_LEN, 1))
    fw = torch.empty(max(fws, 1), dtype=torch.uint8, device=dev)
    bw = torch.empty(bws, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sp, P = rw._stream(stream), rw._ptr

    def fwd(i=0):
        s = h.rwkv_wkv4_forward_gated(B, T, C, rw.F32, P(w), P(u), P(k), P(v), P(r), P(o), None, None, P(ck),
                                      rw.CHUNK_LEN, rw.ALGO_AUTO, P(fw), fws, sp)
        if s:
            raise rw.RwkvError("rwkv_wkv4_forward_gated", s)

    def bwd(i=0):
        s = h.rwkv_wkv4_backward_gated(B, T, C, rw.F32, P(w), P(u), P(k), P(v), P(r), P(go), None, P(ck),
                                       rw.CHUNK_LEN, P(gk), P(gv), P(gr), P(gw), P(gu), P(bw), bws, sp)
        if s:
            raise rw.RwkvError("rwkv_wkv4_backward_gated", s)

    def step(i):
        fwd()
        bwd()

    ms, clk, stats = _timed(step, args.steps, args.warmup, stream, local)
    fwd_ms, _, _ = _timed(fwd, args.steps, args.warmup, stream, local)
    bwd_ms, _, _ = _timed(bwd, args.steps, args.warmup, stream, local)
    rw.rwkv_check_device_error()
    fwd_bytes = 4 * 4 * ELEM                      # k, v, r read; o written
    bwd_bytes = 7 * 4 * ELEM + 2 * 4 * C          # k, v, r, go read; gk, gv, gr written; gw, gu
    peak, kind = _peaks()
    bwd_gbs = bwd_bytes / (bwd_ms * 1e-3) / 1e9
    step_gbs = (fwd_bytes + bwd_bytes) / (ms * 1e-3) / 1e9
    print(json.dumps({
        "metric": "Gated WKV fwd+bwd elements/s and HBM GB/s (o = sigmoid(r) * WKV) at B8 T4096 C2048",
        "value": ELEM / (ms * 1e-3), "unit": "elements/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "RWKV-4 receptance-gated WKV forward+backward, fp32, B=8 T=4096 C=2048, 1% "
                               "+-U(20,40) key outliers, r, go ~ N(0,1)",
                   "l2": "no flush: every input (268 MB each) is larger than the 126 MB L2"},
        "hbm_gbs_step": step_gbs, "hbm_frac_step": step_gbs / peak,
        "kernels_ms": {"wkv4_forward_gated": fwd_ms, "wkv4_backward_gated": bwd_ms},
        "roofline": {"bound": "hbm", "kernel": "wkv4_bwd_kernel<float, gated> (+ its gw/gu batch reduction)",
                     "achieved": bwd_gbs, "peak": peak, "peak_kind": kind, "unit": "GB/s",
                     "frac": bwd_gbs / peak, "traffic": _recorded_traffic("wkv4_bwd_kernel/gated")},
        "gpu_launches": 3 * args.steps, "clocks": clk, "call_ms": stats}), flush=True)


def run_chunked(args):
    """The few-channel forward: B=8 T=1024 C=768 fp32 with 1 % +-U(20,40) key outliers
    (6,144 channel lanes, too few to fill the GPU one thread per lane).  Its 75.5 MB
    fit in the 126 MB L2, so every timed call follows a write of a 256 MB buffer that
    evicts them (cold); back-to-back calls without the flush are reported beside
    (warm).  AUTO (which picks the chunked schedule here), SEQUENTIAL and CHUNKED are
    timed side by side."""
    import torch

    import rwkv_wkv_recurrence_b200 as rw
    import wkv_inputs as wi

    _, _, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    Bc, Tc, Cc = (1, 4096, 768) if args.chunked_shape == "1x4096x768" else (8, 1024, 768)
    p = wi.wkv4_problem(Bc, Tc, Cc, wi.CONFIG_SEED_BASE + 1, outliers=True, device=dev)
    w, u, k, v = p["w"], p["u"], p["k"], p["v"]
    y = torch.empty_like(k)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    h = rw.lib()
    stream = torch.cuda.current_stream()
    sp, P = rw._stream(stream), rw._ptr
    elems = Bc * Tc * Cc
    nbytes = 3 * 4 * elems + 2 * 4 * Cc  # k, v read, y written; w, u
    peak, kind = _peaks()
    names = {rw.ALGO_AUTO: "auto", rw.ALGO_SEQUENTIAL: "sequential", rw.ALGO_CHUNKED: "chunked"}
    res = {}
    clk_all = None
    for algo in (rw.ALGO_AUTO, rw.ALGO_SEQUENTIAL, rw.ALGO_CHUNKED):
        wsb = int(h.rwkv_wkv4_forward_workspace_bytes(Bc, Tc, Cc, algo))
        ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev)

        def call(i=0):
            with _Nvtx("rwkv_wkv4_forward"):
                s = h.rwkv_wkv4_forward(Bc, Tc, Cc, rw.F32, P(w), P(u), P(k), P(v), P(y), None, None, None,
                                        rw.CHUNK_LEN, algo, P(ws), wsb, sp)
            if s:
                raise rw.RwkvError("rwkv_wkv4_forward", s)

        for _ in range(args.warmup):
            call()
        reps = max(20, min(args.steps, 200))
        cold = []
        with ClockSampler(local) as clk:
            torch.cuda.synchronize()
            wall0 = time.perf_counter()
            for _ in range(reps):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                call()
                e1.record(stream)
                e1.synchronize()
                cold.append(e0.elapsed_time(e1))
            clk.mark(wall0, time.perf_counter())
        warm_ms, _, warm = _timed(call, reps, 1, stream, local)
        rw.rwkv_check_device_error()
        st = _stats(cold)
        res[names[algo]] = {"cold_ms": st, "warm_ms": warm, "workspace_bytes": wsb,
                            "cold_gbs_median": nbytes / (st["median"] * 1e-3) / 1e9,
                            "warm_gbs_median": nbytes / (warm["median"] * 1e-3) / 1e9}
        if algo == rw.ALGO_AUTO:
            clk_all = clk.summary()
    auto = res["auto"]["cold_ms"]["median"]
    gbs = nbytes / (auto * 1e-3) / 1e9
    picked = "chunked" if int(h.rwkv_wkv4_forward_workspace_bytes(Bc, Tc, Cc, rw.ALGO_AUTO)) > 0 else "sequential"
    print(json.dumps({
        "metric": f"WKV-4 forward elements/s and HBM GB/s, few channels (B{Bc} T{Tc} C{Cc})",
        "value": elems / (auto * 1e-3), "unit": "elements/s", "n_gpus": 1, "steps": len(res["auto"]["cold_ms"]),
        "warmup": args.warmup, "ms_per_step": auto, "higher_is_better": True, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": f"RWKV-4 WKV forward, fp32, B={Bc} T={Tc} C={Cc}, 1% +-U(20,40) key outliers",
                   "auto_picks": picked,
                   "l2": "flushed: a 256 MB buffer is written before every timed call (inputs fit in L2)"},
        "roofline": {"bound": "hbm", "kernel": f"wkv4_fwd_kernel (AUTO: {picked} schedule)",
                     "achieved": gbs, "peak": peak, "peak_kind": kind, "unit": "GB/s", "frac": gbs / peak,
                     "traffic": None},
        "schedules": res, "gpu_launches": 3 if picked == "chunked" else 1, "clocks": clk_all}), flush=True)


def _omega_range(args):
    lo, hi = (float(x) for x in args.omega_range.split(","))
    if not lo < hi:
        raise SystemExit("--omega-range wants LO,HI with LO < HI")
    return lo, hi


def run_eagle(args, finch=False):
    """Eagle / RWKV-5 forward, B4 T4096 H40 N64 bf16, zero initial state; with
    finch, the Finch / RWKV-6 forward on the same shape with a per-token fp32
    omega [B,T,H,N]."""
    import torch

    import rwkv_wkv_recurrence_b200 as rw
    import wkv_inputs as wi

    _, _, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    Be, Te, He, Ne = 4, 4096, 40, 64
    gen = wi.wkv6_problem if finch else wi.wkv5_problem
    om_lo, om_hi = _omega_range(args)
    q = gen(Be, Te, He, Ne, seed=SEED + (4 if finch else 2), device=dev, omega_range=(om_lo, om_hi))
    y = torch.empty_like(q["r"])
    s_out = torch.empty(Be, He, Ne, Ne, device=dev)
    h = rw.lib()
    stream = torch.cuda.current_stream()
    sp, P = rw._stream(stream), rw._ptr
    fwd = h.rwkv_wkv6_forward if finch else h.rwkv_wkv5_forward
    name = "rwkv_wkv6_forward" if finch else "rwkv_wkv5_forward"
    wsb = int((h.rwkv_wkv6_forward_workspace_bytes if finch else h.rwkv_wkv5_forward_workspace_bytes)(
        Be, Te, He, Ne))
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev)

    def call(i):
        s = fwd(Be, Te, He, Ne, P(q["r"]), P(q["k"]), P(q["v"]), P(q["omega"]), P(q["u"]), P(y), None, P(s_out),
                P(ws), wsb, sp)
        if s:
            raise rw.RwkvError(name, s)

    ms, clk, stats = _timed(call, args.steps, args.warmup, stream, local)
    rw.rwkv_check_device_error()
    elems = Be * Te * He * Ne
    # r, k, v, y bf16; s_out; u (and omega: per token fp32 for Finch, [H,N] fp32 for Eagle)
    nbytes = 4 * 2 * elems + Be * He * Ne * Ne * 4 + He * Ne * 4 + (4 * elems if finch else He * Ne * 4)
    gbs = nbytes / (ms * 1e-3) / 1e9
    peak, kind = _peaks()
    if finch:
        metric = "Finch WKV forward elements/s and HBM GB/s (B4 T4096 H40 N64, per-token decay)"
        workload = ("Finch / RWKV-6 WKV forward, B=4 T=4096 H=40 N=64, bf16 r,k,v,y, fp32 per-token omega "
                    f"(U({om_lo:g},{om_hi:g}) per channel + 0.5 N(0,1) per token), fp32 state")
        l2 = "no flush: 506 MB moved per call, above the 126 MB L2"
        kernel = "wkv6_fwd_tc_kernel"
    else:
        metric = "Eagle WKV forward elements/s and HBM GB/s (B4 T4096 H40 N64)"
        workload = ("Eagle / RWKV-5 WKV forward, B=4 T=4096 H=40 N=64, bf16 r,k,v,y, fp32 state"
                    + ("" if (om_lo, om_hi) == (-6.0, 0.0) else f", omega U({om_lo:g},{om_hi:g})"))
        l2 = "no flush: 338 MB moved per call, above the 126 MB L2"
        kernel = "wkv5_fwd_tc_kernel"
    print(json.dumps({
        "metric": metric, "value": elems / (ms * 1e-3),
        "unit": "elements/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "dtype": "bf16 I/O, fp32 state", "data": "synthetic",
        "config": {"workload": workload, "l2": l2},
        "roofline": {"bound": "hbm", "kernel": kernel, "achieved": gbs, "peak": peak, "peak_kind": kind,
                     "unit": "GB/s", "frac": gbs / peak,
                     # the capture was taken on the default decay range
                     "traffic": _recorded_traffic(kernel) if (om_lo, om_hi) == (-6.0, 0.0) else None},
        "gpu_launches": args.steps, "clocks": clk, "call_ms": stats}), flush=True)


def run_eagle_backward(args, finch=False):
    """Eagle / RWKV-5 backward on the forward workload's shape, B4 T4096 H40 N64 bf16, gy ~ N(0,1),
    zero initial state and no final-state gradient: gr, gk, gv, gomega, gu.  With finch, the
    Finch / RWKV-6 backward on the same shape with a per-token fp32 omega (and a per-token gomega)."""
    import torch

    import rwkv_wkv_recurrence_b200 as rw
    import wkv_inputs as wi

    _, _, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    Be, Te, He, Ne = 4, 4096, 40, 64
    om_lo, om_hi = _omega_range(args)
    gen = wi.wkv6_problem if finch else wi.wkv5_problem
    q = gen(Be, Te, He, Ne, seed=SEED + (4 if finch else 2), device=dev, omega_range=(om_lo, om_hi))
    g = wi.wkv5_grads(Be, Te, He, Ne, seed=SEED + 6, device=dev)
    gr, gk, gv = (torch.empty_like(q["r"]) for _ in range(3))
    gom = torch.empty(Be, Te, He, Ne, device=dev) if finch else torch.empty(He, Ne, device=dev)
    gu = torch.empty(He, Ne, device=dev)
    h = rw.lib()
    name = "rwkv_wkv6_backward" if finch else "rwkv_wkv5_backward"
    fn = getattr(h, name)
    wsb = int(getattr(h, name + "_workspace_bytes")(Be, Te, He, Ne))
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sp, P = rw._stream(stream), rw._ptr

    def call(i):
        with _Nvtx(name):
            s = fn(Be, Te, He, Ne, P(q["r"]), P(q["k"]), P(q["v"]), P(q["omega"]), P(q["u"]), None, P(g["gy"]), None,
                   P(gr), P(gk), P(gv), P(gom), P(gu), None, P(ws), wsb, sp)
        if s:
            raise rw.RwkvError(name, s)

    ms, clk, stats = _timed(call, args.steps, args.warmup, stream, local)
    rw.rwkv_check_device_error()
    elems = Be * Te * He * Ne
    om_note = "" if (om_lo, om_hi) == (-6.0, 0.0) else f", omega U({om_lo:g},{om_hi:g})"
    if finch:
        # r, k, v, gy read and gr, gk, gv written (bf16); omega read and gomega written (fp32, per token)
        nbytes = 7 * 2 * elems + 2 * 4 * elems + 2 * He * Ne * 4
        # algorithmic flops: six N x N multiply-adds per token and head (gr, the state step, gk, gv, the
        # gomega row sums, the gradient-state step), 12 N flops per element; the kernel is bound by the
        # CUDA cores' fp32 issue, so its fraction is taken against the fp32 FMA peak
        flops = 12.0 * Ne * elems
        tf = flops / (ms * 1e-3) / 1e12
        peak_tf = 148 * 128 * 2 * 1.965e9 / 1e12
        metric = "Finch WKV backward elements/s (B4 T4096 H40 N64, per-token decay)"
        workload = ("Finch / RWKV-6 WKV backward, B=4 T=4096 H=40 N=64, bf16 r,k,v,gy,gr,gk,gv, fp32 per-token "
                    "omega and gomega, gy ~ N(0,1), zero initial state, no final-state gradient" + om_note)
        roof = {"bound": "alu", "kernel": "wkv6_bwd_kernel (+ its gu batch reduction)", "achieved": tf,
                "peak": peak_tf, "peak_kind": "derived: 148 SMs x 128 fp32 FMA/clk x 2 flops x 1.965 GHz",
                "unit": "TFLOP/s", "frac": tf / peak_tf, "hbm_gbs": nbytes / (ms * 1e-3) / 1e9,
                # DRAM bytes of one call (its four launches), from the capture on the default decays
                "traffic": _recorded_traffic("rwkv_wkv6_backward") if (om_lo, om_hi) == (-6.0, 0.0) else None}
        l2 = f"no flush: {nbytes / 1e6:.0f} MB moved per call, above the 126 MB L2"
        launches = 2
    else:
        nbytes = 7 * 2 * elems + 4 * He * Ne * 4  # r, k, v, gy read, gr, gk, gv written (bf16); omega, u, gomega, gu
        gbs = nbytes / (ms * 1e-3) / 1e9
        peak, kind = _peaks()
        metric = "Eagle WKV backward elements/s and HBM GB/s (B4 T4096 H40 N64)"
        workload = ("Eagle / RWKV-5 WKV backward, B=4 T=4096 H=40 N=64, bf16 r,k,v,gy,gr,gk,gv, "
                    "gy ~ N(0,1), zero initial state, no final-state gradient" + om_note)
        roof = {"bound": "hbm", "kernel": "rwkv_wkv5_backward (reversed forward + two backward passes + "
                                          "reduction)", "achieved": gbs, "peak": peak, "peak_kind": kind,
                "unit": "GB/s", "frac": gbs / peak,
                "traffic": _recorded_traffic("rwkv_wkv5_backward") if (om_lo, om_hi) == (-6.0, 0.0) else None}
        l2 = "no flush: 587 MB moved per call, above the 126 MB L2"
        launches = 4
    print(json.dumps({
        "metric": metric, "value": elems / (ms * 1e-3),
        "unit": "elements/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "dtype": "bf16 I/O, fp32 state", "data": "synthetic",
        "config": {"workload": workload, "l2": l2}, "roofline": roof,
        "gpu_launches": launches * args.steps, "clocks": clk, "call_ms": stats}), flush=True)


def run_eagle_decode(args, finch=False):
    """Eagle / RWKV-5 decode step: 512 streams x 40 heads x 64, fp32 state
    [512,40,64,64] updated in place, 16 pre-generated bf16 tokens cycled; with
    finch, the Finch / RWKV-6 step with each token's own fp32 omega [512,40,64]."""
    import torch

    import rwkv_wkv_recurrence_b200 as rw
    import wkv_inputs as wi

    _, _, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    Bs, Hs, Ns, Tt = 512, 40, 64, 16
    gen = wi.wkv6_problem if finch else wi.wkv5_problem
    q = gen(Bs, Tt, Hs, Ns, seed=SEED + (7 if finch else 5), device=dev)
    names = ("r", "k", "v", "omega") if finch else ("r", "k", "v")
    toks = [{n: q[n][:, t].contiguous() for n in names} for t in range(Tt)]
    state = torch.zeros(Bs, Hs, Ns, Ns, device=dev)
    y = torch.empty(Bs, Hs, Ns, dtype=torch.bfloat16, device=dev)
    h = rw.lib()
    stream = torch.cuda.current_stream()
    sp, P = rw._stream(stream), rw._ptr

    def step(i):
        t = toks[i % Tt]
        if finch:
            s = h.rwkv_wkv6_step(Bs, Hs, Ns, P(t["r"]), P(t["k"]), P(t["v"]), P(t["omega"]), P(q["u"]), P(y),
                                 P(state), P(state), sp)
        else:
            s = h.rwkv_wkv5_step(Bs, Hs, Ns, P(t["r"]), P(t["k"]), P(t["v"]), P(q["omega"]), P(q["u"]), P(y),
                                 P(state), P(state), sp)
        if s:
            raise rw.RwkvError("rwkv_wkv6_step" if finch else "rwkv_wkv5_step", s)

    ms, clk, stats = _timed(step, args.steps, args.warmup, stream, local)
    heads = Bs * Hs
    # state in + out; r, k, v, y bf16; u (and omega: per stream for Finch, per head for Eagle)
    bytes_step = heads * (2 * Ns * Ns * 4 + 4 * Ns * 2) + Hs * Ns * 4 + (heads * Ns * 4 if finch else Hs * Ns * 4)
    gbs = bytes_step / (ms * 1e-3) / 1e9
    peak, kind = _peaks()
    tag = "Finch" if finch else "Eagle"
    print(json.dumps({
        "metric": f"{tag} decode head-steps/s and HBM GB/s (512 streams x H40 x N64)",
        "value": heads / (ms * 1e-3), "unit": "head-steps/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "dtype": "bf16 I/O, fp32 state",
        "data": "synthetic",
        "config": {"workload": (f"{tag} / RWKV-{6 if finch else 5} decode step, 512 streams x H=40 x N=64, fp32 "
                                f"state in place, 16 tokens cycled" + (", per-token fp32 omega" if finch else "")),
                   "l2": f"no flush: {bytes_step / 1e6:.0f} MB moved per step, above the 126 MB L2"},
        "roofline": {"bound": "hbm", "kernel": "wkv5_step_kernel", "achieved": gbs, "peak": peak,
                     "peak_kind": kind, "unit": "GB/s", "frac": gbs / peak,
                     "traffic": _recorded_traffic("wkv5_step_kernel/finch" if finch else "wkv5_step_kernel")},
        "gpu_launches": args.steps, "clocks": clk, "call_ms": stats}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["train", "train_gated", "decode", "chunked", "eagle", "eagle_bwd",
                                           "eagle_decode", "finch", "finch_bwd", "finch_decode"],
                    default="train",
                    help="train: the headline forward+backward step; train_gated, decode, chunked, eagle, "
                         "eagle_bwd, eagle_decode, finch, finch_bwd, finch_decode: the other hot-path rows")
    ap.add_argument("--chunked-shape", choices=["8x1024x768", "1x4096x768"], default="8x1024x768",
                    help="the few-channel forward's shape (chunked workload)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--omega-range", default="-6,0",
                    help="eagle / finch workloads: the per-channel omega range U(LO,HI) (w = exp(-exp(omega)))")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-channels", type=int, default=256)
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per backward launch, if captured for this kernel version")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "decode":
        run_decode(args)
    elif args.workload == "chunked":
        run_chunked(args)
    elif args.workload == "train_gated":
        run_train_gated(args)
    elif args.workload == "eagle":
        run_eagle(args)
    elif args.workload == "eagle_bwd":
        run_eagle_backward(args)
    elif args.workload == "eagle_decode":
        run_eagle_decode(args)
    elif args.workload == "finch":
        run_eagle(args, finch=True)
    elif args.workload == "finch_bwd":
        run_eagle_backward(args, finch=True)
    elif args.workload == "finch_decode":
        run_eagle_decode(args, finch=True)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
