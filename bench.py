"""Benchmark of the GR-KAN hot path on B200: one step = forward (y) + backward
(dx, then dA / dB through the two-stage reduction) over one batch of
synthetic KAT-shaped activations resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config kat_b]
    python bench.py --impl reference ...      # the fp64 oracle on host cores

Prints one JSON line (rank 0). For N > 1 launch with torchrun; every rank
processes its own batch (weak scaling) and the per-rank float64 gradient sums
are all-gathered over NCCL and merged in rank order.
"""
import argparse
import json
import os
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
from group_rational_kan_b200 import accounting  # noqa: E402

METRIC = "GR-KAN fwd+bwd elements/s and achieved HBM GB/s vs B200 peak (1 GPU)"
UNIT = "elements/s"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="kat_b", choices=list(synth.WORKLOADS))
    ap.add_argument("--ng", type=int, default=None, help="groups for the stress workload")
    ap.add_argument("--rows", type=int, default=None,
                    help="use only the first ROWS rows of the workload (profiling captures)")
    ap.add_argument("--m", type=int, default=None, help="numerator degree (degree sweeps)")
    ap.add_argument("--n", type=int, default=None, help="denominator degree (degree sweeps)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--ref-budget", type=float, default=120.0,
                    help="seconds of oracle work for the whole --impl reference run")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fused-launches", type=int, default=50,
                    help="launches of the recompute variant timed after the step (0: skip)")
    ap.add_argument("--linear-nout", type=int, default=768,
                    help="also time the activation fused into a following linear layer with "
                         "this many outputs (bf16 workloads; default 768, the KAT-B MLP's "
                         "second linear layer; 0: skip)")
    ap.add_argument("--per-config", default="kat_t,kat_s,stress:1,stress:8,stress:64",
                    help="other workloads timed after the main step (name[:n_g], comma "
                         "separated; empty: skip)")
    ap.add_argument("--per-config-steps", type=int, default=20)
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s, earlier measurement on this pool)"


def tensor_peak():
    """Dense bf16 tensor-core peak (TFLOP/s) for a kernel timed alone: the
    measured burst cuBLAS figure, else the fallback measurement."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, burst)"
    except Exception:
        return 1590.0, "fallback (1.59 PFLOP/s, earlier measurement on this pool)"


def measured_traffic(w):
    """DRAM bytes per backward launch from the committed ncu summary, scaled by
    elements; None unless the summary covers this workload and the kernel
    sources are the ones it was captured on."""
    import hashlib
    if w.name != "kat_b":
        return None
    try:
        text = open(os.path.join(ROOT, "profiles", "bwd_tma_kat_b.md")).read()
        per = float(text.split("traffic_bytes_per_element:")[1].split()[0])
        want = text.split("kernel_source_sha256_16:")[1].split()[0]
        h = hashlib.sha256()
        for f in ("grkan_tma.cuh", "grkan_common.cuh"):
            h.update(open(os.path.join(ROOT, "group_rational_kan_b200", "csrc", f), "rb").read())
        if h.hexdigest()[:16] != want:
            return None
        return per * w.elems
    except Exception:
        return None


def dtype_name(w):
    return "f32" if w.dtype == synth.F32 else "bf16"


# --- clocks ---------------------------------------------------------------------

class ClockSampler:
    """SM clock and throttle reasons sampled during the timed region: through NVML
    every 2 ms in a background thread when the bindings are there (a timed region
    of a few milliseconds still gets several samples), else `nvidia-smi -lms 100`.
    Read-only: nothing here changes a setting of the GPU."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_id, interval_s=0.002):
        self.gpu_id = gpu_id
        self.interval = interval_s
        self.proc = None
        self.thread = None
        self.path = os.path.join(tempfile.gettempdir(), "grkan_clocks_%d.csv" % os.getpid())

    def _nvml_loop(self, nv, h, bits):
        sm, mx, reasons = [], [], set()
        maxc = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        self.t_first = self.t_last = None
        while not self.stop_flag.is_set():
            try:
                now = time.perf_counter()
                self.t_first = now if self.t_first is None else self.t_first
                self.t_last = now
                sm.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                mx.append(float(maxc))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                for name, bit in bits.items():
                    if r & bit:
                        reasons.add(name)
            except Exception:
                pass
            self.ready.set()
            self.stop_flag.wait(self.interval)
        self.ready.set()
        self.result = (sm, mx, reasons)

    def start(self):
        try:
            import threading
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByUUID(self.gpu_id)
            bits = {"hw_slowdown": nv.nvmlClocksThrottleReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksThrottleReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksThrottleReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksThrottleReasonSwPowerCap}
            self.stop_flag = threading.Event()
            self.ready = threading.Event()
            self.result = None
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h, bits),
                                           daemon=True)
            self.thread.start()
            self.ready.wait(2.0)  # sampling before the timed region starts
            self.source = "nvml, every %.0f ms" % (self.interval * 1e3)
            return
        except Exception:
            self.thread = None
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi, every 100 ms"
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def _summary(self, sm, mx, reasons):
        if not sm:
            return None
        out = {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)),
               "samples": len(sm), "reasons": sorted(reasons), "source": self.source}
        if getattr(self, "t_first", None) is not None:
            out["window_ms"] = (self.t_last - self.t_first) * 1e3
        return out

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            return self._summary(*self.result) if self.result else None
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(self.REASONS, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return self._summary(sm, mx, reasons)


# --- reference arm / CPU baseline: the fp64 oracle on host cores ----------------------

def oracle_step(orc, w, x, dy, a, b):
    orc.forward(x, a, b, w.n_g)
    orc.backward_elem(x, dy, a, b, w.n_g)
    orc.coef_grads(x, dy, a, b, w.n_g)


def oracle_rate(w, target_s, min_rows=1):
    """Time the oracle (as it stands) on the first rows of the workload."""
    import oracle
    orc = oracle.Oracle()
    rows = max(min_rows, 1)
    while True:
        s = w.with_rows(rows)
        x, dy = s.x(), s.dy()
        a, b = s.coefficients()
        t0 = time.perf_counter()
        oracle_step(orc, s, x, dy, a, b)
        dt = time.perf_counter() - t0
        if dt >= target_s or rows >= w.rows:
            return rows, dt, orc.max_threads()
        rows = min(w.rows, max(rows * 2, int(rows * target_s / max(dt, 1e-3) * 1.05)))


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    orc = oracle.Oracle()
    # size one step so that warmup + steps take about --ref-budget seconds in all
    budget = args.ref_budget / max(args.steps + args.warmup, 1)
    rows, dt, cores = oracle_rate(w, min(budget, 2.0))
    per_row = dt / rows
    rows = max(1, min(w.rows, int(budget / per_row)))
    s = w.with_rows(rows)
    x, dy = s.x(), s.dy()
    a, b = s.coefficients()
    for _ in range(args.warmup):
        oracle_step(orc, s, x, dy, a, b)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(orc, s, x, dy, a, b)
    el = time.perf_counter() - t0
    value = s.elems * args.steps / el
    sample = "first %d of %d rows of %s per step (%d elements), fwd y + bwd dx + dA/dB" % (
        rows, w.rows, w.name, s.elems)
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(w.describe(), global_batch=w.B * args.gpus, seq_len=w.N,
                       parallelism="dp%d" % args.gpus,
                       l2="host memory; each step a bounded sample of the workload",
                       rows_per_step=rows),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


# --- other workloads, timed after the main step ----------------------------------------

def time_workload(grk, torch, dev, w, steps, peak):
    """Forward, backward and step times of one workload on device-resident inputs
    (CUDA events per kernel, medians over `steps` steps after 3 warm-ups), plus
    the one-pass forward + backward."""
    B, N, d, n_g, m, n, dt = w.B, w.N, w.d, w.n_g, w.m, w.n, w.dtype
    E = w.elems
    tdt = torch.float32 if dt == synth.F32 else torch.bfloat16
    xh = torch.empty((B, N, d), dtype=tdt, pin_memory=True)
    gh = torch.empty((B, N, d), dtype=tdt, pin_memory=True)
    synth.fill_ptr(xh.data_ptr(), E, dt, w.seed, synth.X_STREAM, w.x_kind, w.x_scale, w.x_clip)
    synth.fill_ptr(gh.data_ptr(), E, dt, w.seed, synth.DY_STREAM, synth.KIND_NORMAL, w.dy_scale)
    x, dy = xh.to(dev), gh.to(dev)
    del xh, gh
    a_np, b_np = w.coefficients()
    a, b = torch.from_numpy(a_np).to(dev), torch.from_numpy(b_np).to(dev)
    y, dx = torch.empty_like(x), torch.empty_like(x)
    dA = torch.empty((n_g, m + 1), dtype=torch.float32, device=dev)
    dB = torch.empty((n_g, n), dtype=torch.float32, device=dev)
    wsb = grk.grkan_backward_workspace_bytes(B, N, d, n_g, m, n, dt)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream

    def ok(st, what):
        if st != 0:
            raise grk.GrkanError(st, what)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        ok(grk.grkan_forward(x, y, a, b, B, N, d, n_g, m, n, dt, sp), "forward")
        if ev is not None:
            ev[1].record(stream)
        ok(grk.grkan_backward_partials(x, dy, a, b, dx, B, N, d, n_g, m, n, dt, ws, wsb, 0, sp),
           "backward_partials")
        if ev is not None:
            ev[2].record(stream)
        ok(grk.grkan_backward_merge(ws, wsb, dA, dB, None, B, N, d, n_g, m, n, dt, sp), "merge")
        if ev is not None:
            ev[3].record(stream)

    for _ in range(3):
        step()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for k in range(steps):
        step(evs[k])
    torch.cuda.synchronize(dev)
    fwd = float(np.median([e[0].elapsed_time(e[1]) for e in evs]))
    bwd = float(np.median([e[1].elapsed_time(e[2]) for e in evs]))
    stp = float(np.median([e[0].elapsed_time(e[3]) for e in evs]))

    def one_pass():
        ok(grk.grkan_forward_backward(x, dy, a, b, y, dx, dA, dB, B, N, d, n_g, m, n, dt, ws, wsb,
                                      0, sp), "forward_backward")
    for _ in range(3):
        one_pass()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(steps):
        one_pass()
    f1.record(stream)
    torch.cuda.synchronize(dev)
    fb = f0.elapsed_time(f1) / steps

    def rates(kind, ms):
        by = accounting.bytes_per_element(kind, dt) * E
        return {"ms": ms, "GB/s": by / (ms * 1e-3) / 1e9, "frac": by / (ms * 1e-3) / 1e9 / peak,
                "frac_of_8TBps": by / (ms * 1e-3) / 8e12}
    out = {"workload": w.name, "dtype": dtype_name(w), "shape": [B, N, d], "n_g": n_g,
           "elements": E, "elements_per_s": E / (stp * 1e-3),
           "forward": rates("forward", fwd), "backward_stage1": rates("backward", bwd),
           "step": rates("step", stp), "forward_backward_recompute": rates("forward_backward", fb),
           "kernel_path": {"forward": "tma" if grk.grkan_forward_path(
               x, y, B, N, d, n_g, m, n, dt) == 1 else "generic",
               "backward": "tma" if grk.grkan_backward_path(
               x, dy, dx, B, N, d, n_g, m, n, dt) == 1 else "generic"}}
    del x, dy, y, dx, ws
    torch.cuda.empty_cache()
    return out


# --- our arm ---------------------------------------------------------------------------

def main():
    args = parse()
    w = synth.workload(args.config, n_g=args.ng)
    if args.rows is not None:
        w = w.with_rows(args.rows)
        w.B, w.N = args.rows, 1
        w.rows_override = None
    if args.m is not None:
        w.m = args.m
    if args.n is not None:
        w.n = args.n
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import torch.distributed as dist
    import group_rational_kan_b200 as grk
    from group_rational_kan_b200.dist import all_gather_sums

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    w.seed = rank  # weak scaling: every rank its own batch
    B, N, d, n_g, m, n, dt = w.B, w.N, w.d, w.n_g, w.m, w.n, w.dtype
    E = w.elems
    es = w.es
    tdt = torch.float32 if dt == synth.F32 else torch.bfloat16
    nbytes = E * es

    # inputs: generated on the host into pinned memory, then copied to HBM
    x_h = torch.empty((B, N, d), dtype=tdt, pin_memory=True)
    dy_h = torch.empty((B, N, d), dtype=tdt, pin_memory=True)
    synth.fill_ptr(x_h.data_ptr(), E, dt, w.seed, synth.X_STREAM, w.x_kind, w.x_scale, w.x_clip)
    synth.fill_ptr(dy_h.data_ptr(), E, dt, w.seed, synth.DY_STREAM, synth.KIND_NORMAL, w.dy_scale)
    a_np, b_np = w.coefficients()
    a = torch.from_numpy(a_np).to(dev)
    b = torch.from_numpy(b_np).to(dev)
    x = x_h.to(dev)
    dy = dy_h.to(dev)
    y = torch.empty_like(x)
    dx = torch.empty_like(x)
    dA = torch.empty((n_g, m + 1), dtype=torch.float32, device=dev)
    dB = torch.empty((n_g, n), dtype=torch.float32, device=dev)
    wsb = grk.grkan_backward_workspace_bytes(B, N, d, n_g, m, n, dt)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    K = m + 1 + n
    sums64 = torch.empty((n_g, K), dtype=torch.float64, device=dev) if world > 1 else None
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    path_f = grk.grkan_forward_path(x, y, B, N, d, n_g, m, n, dt)
    path_b = grk.grkan_backward_path(x, dy, dx, B, N, d, n_g, m, n, dt)

    def check(st, what):
        if st != 0:
            raise grk.GrkanError(st, what)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        check(grk.grkan_forward(x, y, a, b, B, N, d, n_g, m, n, dt, sp), "forward")
        if ev is not None:
            ev[1].record(stream)
        check(grk.grkan_backward_partials(x, dy, a, b, dx, B, N, d, n_g, m, n, dt, ws, wsb, 0, sp),
              "backward_partials")
        if ev is not None:
            ev[2].record(stream)
        check(grk.grkan_backward_merge(ws, wsb, dA, dB, sums64, B, N, d, n_g, m, n, dt, sp),
              "backward_merge")
        if world > 1:
            g = all_gather_sums(sums64)
            check(grk.grkan_merge_ranks(g, world, dA, dB, n_g, m, n, sp), "merge_ranks")

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    grads_warm = torch.cat([dA.flatten(), dB.flatten()]).clone()

    # timed region: exactly K steps between a barrier + synchronize on each side
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler("GPU-" + str(props.uuid))
    sampler.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_start.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t_end.record(stream)
    # wait for the end event while letting the clock sampler's thread run (a
    # blocking synchronize can hold the interpreter for the whole timed region)
    while not t_end.query():
        time.sleep(0.0005)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    # dA / dB after the last timed step against the copy taken after warm-up:
    # the two-stage reduction gives the same bits every step
    grads_last = torch.cat([dA.flatten(), dB.flatten()])
    import hashlib
    determinism = {
        "dA_dB_identical_over_steps": bool(torch.equal(grads_warm, grads_last)),
        "dA_dB_sha256_16": hashlib.sha256(
            grads_last.cpu().numpy().tobytes()).hexdigest()[:16]}
    ms_total = t_start.elapsed_time(t_end)
    fwd_all = [e[0].elapsed_time(e[1]) for e in evs]
    bwd_all = [e[1].elapsed_time(e[2]) for e in evs]
    fwd_ms = float(np.mean(fwd_all))
    bwd_ms = float(np.mean(bwd_all))
    if world > 1:
        t = torch.tensor([ms_total], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_total = float(t.item())
    ms_step = ms_total / args.steps
    value = E * world / (ms_step * 1e-3)

    # the recompute variant (y rewritten inside the backward pass, for activation
    # checkpointing), outside the timed step: reported for information only
    fused_ms = None
    if args.fused_launches > 0:
        def fused():
            check(grk.grkan_forward_backward(x, dy, a, b, y, dx, dA, dB, B, N, d, n_g, m, n, dt,
                                             ws, wsb, 0, sp), "forward_backward")
        for _ in range(3):
            fused()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.fused_launches):
            fused()
        f1.record(stream)
        torch.cuda.synchronize(dev)
        fused_ms = f0.elapsed_time(f1) / args.fused_launches

    # the activation fused into a following linear layer (bf16 only), outside the
    # timed step: fused kernel against the activation kernel plus cuBLAS
    linear = None
    if args.linear_nout > 0 and dt == synth.BF16 and (m, n) == (5, 4):
        nout = args.linear_nout
        gen = torch.Generator(device=dev).manual_seed(1234 + rank)
        Wl = (torch.randn(nout, d, device=dev, generator=gen) / d ** 0.5).to(torch.bfloat16)
        outl = torch.empty((B * N, nout), dtype=torch.bfloat16, device=dev)

        def lin_fused():
            check(grk.grkan_linear_forward(x, a, b, Wl, None, outl, B, N, d, n_g, m, n, nout, dt,
                                           sp), "linear_forward")

        def lin_unfused():
            check(grk.grkan_forward(x, y, a, b, B, N, d, n_g, m, n, dt, sp), "forward")
            torch.matmul(y.view(B * N, d), Wl.t(), out=outl)

        def timed(f, k=20):
            for _ in range(3):
                f()
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for _ in range(k):
                f()
            t1.record(stream)
            torch.cuda.synchronize(dev)
            return t0.elapsed_time(t1) / k

        fl = 2.0 * B * N * d * nout
        tpeak, tsrc = tensor_peak()

        def tensor_roofline(ms):
            ach = fl / (ms * 1e-3) / 1e12
            return {"bound": "tensor", "achieved": ach, "peak": tpeak, "unit": "TFLOP/s",
                    "frac": ach / tpeak, "peak_source": tsrc,
                    "flops_per_launch": fl}

        # alternated three times, medians
        ff, uf = [], []
        for _ in range(3):
            ff.append(timed(lin_fused))
            uf.append(timed(lin_unfused))
        f_ms, u_ms = sorted(ff)[1], sorted(uf)[1]
        path = grk.grkan_linear_forward_path(B, N, d, n_g, m, n, nout, dt)
        linear = {"nout": nout, "fused_ms": f_ms, "unfused_ms": u_ms,
                  "fused_TFLOP/s": fl / (f_ms * 1e-3) / 1e12,
                  "roofline": tensor_roofline(f_ms),
                  "kernel": {1: "clusters of four CTAs", 0: "one CTA per tile"}.get(path, path),
                  "note": "grkan_linear_forward vs grkan_forward + torch.matmul (cuBLAS), "
                          "no bias; not part of the timed step"}

        # its backward: dy = dout W on the tensor cores with the GR-KAN backward as
        # the epilogue, against torch.matmul (cuBLAS, bf16 dy) + grkan_backward;
        # alternated three times, medians
        dout = (torch.randn(B * N, nout, device=dev, generator=gen) * 1e-2).to(torch.bfloat16)
        dyl = torch.empty_like(dy)
        wslb = grk.grkan_linear_backward_workspace_bytes(B, N, d, n_g, m, n, nout, dt)
        wsl = torch.empty(max(wslb, 16), dtype=torch.uint8, device=dev)

        def lbw_fused():
            check(grk.grkan_linear_backward(x, dout, Wl, a, b, dx, dA, dB, B, N, d, n_g, m, n,
                                            nout, dt, wsl, wslb, sp), "linear_backward")

        def lbw_unfused():
            torch.matmul(dout, Wl, out=dyl.view(B * N, d))
            check(grk.grkan_backward(x, dyl, a, b, dx, dA, dB, B, N, d, n_g, m, n, dt, ws, wsb,
                                     sp), "backward")

        fb, ub = [], []
        for _ in range(3):
            fb.append(timed(lbw_fused))
            ub.append(timed(lbw_unfused))
        fb_ms, ub_ms = sorted(fb)[1], sorted(ub)[1]
        linear["backward"] = {
            "fused_ms": fb_ms, "unfused_ms": ub_ms,
            "fused_TFLOP/s": fl / (fb_ms * 1e-3) / 1e12,
            "roofline": tensor_roofline(fb_ms),
            "note": "grkan_linear_backward (dout W + GR-KAN backward epilogue, CTA pairs) vs "
                    "torch.matmul (cuBLAS) + grkan_backward; weight gradient not included"}
        del Wl, outl, dout, dyl, wsl

    # the other workloads (KAT-T, KAT-S, the group stress sweep), each timed on its
    # own device-resident inputs after the main step; not part of `value`
    per_config = None
    if args.per_config and world == 1:
        peak_gbs = peaks()[0]
        per_config = []
        for item in [c for c in args.per_config.split(",") if c]:
            cname, _, cng = item.partition(":")
            cw = synth.workload(cname, n_g=int(cng) if cng else None)
            per_config.append(time_workload(grk, torch, dev, cw, args.per_config_steps,
                                            peak_gbs))

    # end to end through the C ABI's host-buffer entry point: pinned inputs in,
    # y, dx and dA/dB out, copies inside the timed region (chunks streamed over
    # three streams so that copies in, kernels and copies out overlap)
    y_h = torch.empty_like(x_h, pin_memory=True)
    dx_h = torch.empty_like(x_h, pin_memory=True)
    dA_h = torch.empty(dA.shape, dtype=torch.float32, pin_memory=True)
    dB_h = torch.empty(dB.shape, dtype=torch.float32, pin_memory=True)
    del x, dy, y, dx  # the host path stages its own chunks
    torch.cuda.empty_cache()
    sneed = grk.grkan_step_host_scratch_bytes(B, N, d, n_g, m, n, dt, 0)
    scratch = torch.empty(sneed, dtype=torch.uint8, device=dev)

    def e2e_step():
        # at N > 1 the step also leaves this rank's float64 sums on the device; the
        # ranks exchange them and merge in rank order, then the gradients go to
        # the host (the same bits on every rank)
        check(grk.grkan_step_host(x_h, dy_h, a, b, y_h, dx_h, dA_h, dB_h, sums64, B, N, d, n_g,
                                  m, n, dt, scratch, sneed, 0, sp), "step_host")
        if world > 1:
            g = all_gather_sums(sums64)
            check(grk.grkan_merge_ranks(g, world, dA, dB, n_g, m, n, sp), "merge_ranks")
            dA_h.copy_(dA, non_blocking=True)
            dB_h.copy_(dB, non_blocking=True)

    for _ in range(min(2, args.e2e_steps)):
        e2e_step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / max(args.e2e_steps, 1)
    if world > 1:
        t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    st, derr = grk.grkan_device_error()

    peak, peak_src = peaks()
    bwd_bytes = accounting.bytes_per_element("backward", dt) * E
    fwd_bytes = accounting.bytes_per_element("forward", dt) * E
    step_bytes = accounting.bytes_per_element("step", dt) * E
    fused_bytes = accounting.bytes_per_element("forward_backward", dt) * E
    achieved = bwd_bytes / (bwd_ms * 1e-3) / 1e9
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    clk = clocks or {}
    clk_mhz = float(clk.get("sm_mhz") or clk.get("sm_max_mhz") or 1965.0)
    alu_ops = accounting.backward_fma_ops_per_element(m, n) * E
    alu_peak = accounting.fma_pipe_peak(sms, clk_mhz)
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "dtype_note": "arithmetic type of the kernels (float32, float64 merge); the "
                      "workload's tensors are config.dtype (%s)" % dtype_name(w),
        "data": "synthetic (seeded counter-based generator; KAT activation shapes)",
        "config": dict(w.describe(), global_batch=B * world, seq_len=N,
                       parallelism="dp%d" % world,
                       l2="inputs larger than L2 (%.0f MB per tensor), no flush" % (nbytes / 1e6),
                       kernel_path={"forward": "tma" if path_f == 1 else "generic",
                                    "backward": "tma" if path_b == 1 else "generic"}),
        "roofline": {"bound": "hbm", "kernel": "backward stage 1 (dx + dA/dB partials)",
                     "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": measured_traffic(w),
                     "traffic_note": "ncu dram__bytes_read + dram__bytes_write of one launch "
                                     "on the first 25,000 rows, scaled by elements "
                                     "(profiles/bwd_tma_kat_b.md): reads equal the "
                                     "algorithmic x + dy bytes; writes come out below the "
                                     "algorithmic dx bytes because the capture's last dx "
                                     "lines are still in L2 when the kernel ends",
                     "peak_source": peak_src,
                     "bytes_per_launch": bwd_bytes, "launch_ms": bwd_ms},
        # the backward kernel is bound by FP32 arithmetic, not HBM: the same
        # launch against the FMA pipe's peak at the median SM clock seen under load
        "roofline_alu": {
            "bound": "alu", "kernel": "backward stage 1 (dx + dA/dB partials)",
            "achieved": alu_ops / (bwd_ms * 1e-3) / 1e9, "peak": alu_peak / 1e9,
            "unit": "Gop/s", "frac": alu_ops / (bwd_ms * 1e-3) / alu_peak,
            "ops_per_element": accounting.backward_fma_ops_per_element(m, n),
            "peak_source": "128 FMA-pipe lane operations per SM-cycle x %d SMs x %.0f MHz "
                           "(median SM clock during the timed region)" % (sms, clk_mhz)},
        "kernels": {
            "forward": {"ms": fwd_ms, "GB/s": fwd_bytes / (fwd_ms * 1e-3) / 1e9,
                        "frac": fwd_bytes / (fwd_ms * 1e-3) / 1e9 / peak,
                        "frac_of_8TBps": fwd_bytes / (fwd_ms * 1e-3) / 8e12,
                        "ms_median": float(np.median(fwd_all)), "ms_best": float(min(fwd_all))},
            "backward_stage1": {"ms": bwd_ms, "GB/s": achieved, "frac": achieved / peak,
                                "frac_of_8TBps": bwd_bytes / (bwd_ms * 1e-3) / 8e12,
                                "ms_median": float(np.median(bwd_all)),
                                "ms_best": float(min(bwd_all))},
            "forward_backward_recompute": None if fused_ms is None else {
                "ms": fused_ms, "GB/s": fused_bytes / (fused_ms * 1e-3) / 1e9,
                "frac": fused_bytes / (fused_ms * 1e-3) / 1e9 / peak,
                "frac_of_8TBps": fused_bytes / (fused_ms * 1e-3) / 8e12,
                "note": "y, dx and dA/dB from one pass over x and dy (4 element sizes per "
                        "element), merge included; activation-recompute training only, not "
                        "part of the timed step"},
            "step": {"ms": ms_step, "GB/s": step_bytes / (ms_step * 1e-3) / 1e9,
                     "frac": step_bytes / (ms_step * 1e-3) / 1e9 / peak,
                     "frac_of_8TBps": step_bytes / (ms_step * 1e-3) / 8e12},
        },
        "e2e": {"value": E * world / (e2e_ms * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": 2 * nbytes,
                "d2h_bytes_per_step": 2 * nbytes + (n_g * K) * 4, "ms_per_step": e2e_ms,
                "api": "grkan_step_host (x, dy in; y, dx, dA, dB out; pinned host buffers)"},
        "fused_linear": linear,
        "per_config": per_config,
        "determinism": determinism,
        "gpu_launches": args.steps * (3 + (1 if world > 1 else 0)),
        "clocks": clocks,
        "device_error": derr,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows, el, cores = oracle_rate(w, args.cpu_seconds)
        s_el = rows * w.d
        out["cpu_baseline"] = {
            "value": s_el / el, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": "first %d of %d rows of %s (%d elements), fwd y + bwd dx + dA/dB, %.1f s"
                      % (rows, w.rows, w.name, s_el, el)}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
