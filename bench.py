"""Benchmark of the ternary decode GEMV hot path on B200.

Workload (one "step"): the 8B-class decode layer set at batch 1 in both packed layouts — GEMVs
N x K = 4096 x 4096 (attention projection), 24576 x 4096 (fused gate/up), 4096 x 12288 (down),
each in Q2_0_g128 and in base-3 (5 trits/byte) — and the LM head 151936 x 4096 in base-3 at batch 1,
i.e. seven tern_gemv calls per step. Inputs are seeded synthetic codes (P(0)=0.4, P(+-1)=0.3), scales
fp16(|N(0,1)|*0.02), activations fp16(N(0,1)).
Metric: algorithmic bytes (packed codes + fp16 scales + x + y) per second, GB/s, whole job.

L2 policy: the step rotates over enough copies of the weights that the footprint exceeds 3x the
L2 size, so every step reads its weights from HBM. Device time comes from CUDA events on the
launching stream around exactly --steps graph replays, with a barrier + synchronize on both sides
and the max over ranks. Multi-GPU runs are independent replicas (weak scaling, no data-path
collective). The e2e figure repeats the step through the public API with host-resident
activations (pinned) copied in and results copied out inside the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--no-extras]
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

LAYER_SET = [(4096, 4096), (24576, 4096), (4096, 12288)]  # (N, K) of the 8B-class decode layers
LM_HEAD = (151936, 4096)  # (N, K) of the LM head (base-3 layout)
GROUP = 128
L2_BYTES_DEFAULT = 126 * 1024 * 1024
METRIC = "ternary GEMV GB/s (weights/s) & % of 8 TB/s HBM; GEMM TFLOP/s vs fp16 peak"
WORKLOAD = ("8B-class decode layer set (Q2_0_g128 + base-3: 4096x4096, 24576x4096, 4096x12288) and the "
            "LM head 151936x4096 (base-3), batch 1")


def _env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=12000)
    p.add_argument("--warmup", type=int, default=50)
    p.add_argument("--impl", default="native", choices=["native", "reference"])
    p.add_argument("--no-extras", action="store_true", help="skip the per-row measurements of the other kernels")
    p.add_argument("--eager", action="store_true",
                   help="launch each step's GEMVs directly instead of replaying the step's CUDA graph (the same "
                        "kernels and arguments; used for the ncu launch list, whose per-kernel replay of graph "
                        "nodes does not launch the thread-block-cluster kernels)")
    p.add_argument("--profile", default=None, metavar="CASE",
                   help="run a few launches of one kernel case for ncu: gemv_{q2|t3|q1}_NxK_bB, "
                        "gemm_{q2|t3|q1}_MxNxK, pack_{q2|t3|q1}_NxK, unpack_{q2|t3|q1}_NxK, "
                        "gemvt_{q2|t3|q1}_NxK_bB, rotate_bB_kK; or 'all' for one case of every kernel")
    p.add_argument("--record-traffic", default=None, metavar="NCU_CSV",
                   help="write profiles/traffic.json from an ncu --csv capture of the dominant GEMV "
                        "(dram__bytes_read.sum + dram__bytes_write.sum), keyed by the current source digest")
    return p.parse_args()


# ------------------------------------------------------------------------------------- helpers
def algorithmic_bytes(layout: int, n: int, k: int, batch: int) -> int:
    """Bytes a GEMV must move: packed code rows + k/128 fp16 scales per row + x + y."""
    import gemm_tern_gemv_b200 as T
    return n * T.row_bytes(layout, k) + n * (k // GROUP) * 2 + batch * k * 2 + batch * n * 2


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def source_digest(name: str) -> str:
    import hashlib
    with open(os.path.join(ROOT, "gemm_tern_gemv_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(kernel_key: str):
    """dram bytes per launch from the committed ncu summary, if taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[kernel_key]
        if e.get("source_sha") == source_digest(e["source"]):
            return e["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


class ClockSampler:
    """Samples the SM clock, power and clock-event (throttle) reasons of one GPU while the timed region
    runs; only samples taken between begin() and end() enter the summary. NVML is polled every 2 ms
    from a thread (so even a short region gets samples); without NVML, `nvidia-smi -lms 200` is read."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, index: int, pci_bus_id: str | None = None):
        self.index = index
        self.pci = pci_bus_id
        self.rows = []  # (host time, sm MHz, max sm MHz, power W, reason names)
        self.proc = None
        self.thread = None
        self.stop = threading.Event()
        self.source = None
        self.t0 = self.t1 = None
        self._sample = None

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = None
            if self.pci:
                try:
                    h = nv.nvmlDeviceGetHandleByPciBusId(self.pci)
                except Exception:
                    h = None
            if h is None:
                h = nv.nvmlDeviceGetHandleByIndex(self.index)
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown | nv.nvmlClocksEventReasonHwPowerBrakeSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))

            def one():
                try:
                    sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.rows.append((time.time(), sm, mx, pw, [k for k, b in bits.items() if r & b]))
                except Exception:
                    pass

            def poll():
                while not self.stop.is_set():
                    one()
                    time.sleep(0.002)

            self._sample = one

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            self.source = "nvml, 2 ms polling"
            return self
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            self.source = "nvidia-smi -lms 200"
            deadline = time.time() + 5.0  # nvidia-smi takes a moment to print its first sample
            while not self.rows and time.time() < deadline and self.proc.poll() is None:
                time.sleep(0.02)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                names = [self.NAMES[i] for i in range(4) if parts[5 + i].lower() == "active"]
                self.rows.append((time.time(), num(parts[1]), num(parts[2]), num(parts[3]), names))

    def sample_now(self):
        """One synchronous sample (NVML only), taken while the GPU runs the timed work."""
        if self._sample is not None:
            self._sample()

    def begin(self):
        self.t0 = time.time()

    def end(self):
        self.t1 = time.time()

    def __exit__(self, *exc):
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        rows = [r for r in list(self.rows)
                if self.t0 is not None and self.t1 is not None and self.t0 <= r[0] <= self.t1]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        sm = [r[1] for r in rows if r[1] is not None]
        mx = [r[2] for r in rows if r[2] is not None]
        pw = [r[3] for r in rows if r[3] is not None]
        reasons = sorted({n for r in rows for n in r[4]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "power_w_median": statistics.median(pw) if pw else None,
                "source": self.source}


# ----------------------------------------------------------------------------- the native arm
def make_weights(torch, T, n, k, layout, seed, device):
    """Seeded synthetic packed weights generated on the device and packed with tern_pack."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    u = torch.rand((n, k), generator=g, device=device)
    t = torch.where(u < 0.3, -1.0, torch.where(u < 0.7, 0.0, 1.0))
    s = (torch.randn((n, k // GROUP), generator=g, device=device).abs() * 0.02).to(torch.float16)
    w = (t * s.float().repeat_interleave(GROUP, dim=1)).to(torch.float16)  # exact: s * t
    del u, t
    return T.pack(w, s, layout)


def run_native(args, rank, world, local_rank):
    import torch
    import gemm_tern_gemv_b200 as T

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    T.lib()
    peaks = load_peaks()
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", L2_BYTES_DEFAULT) or L2_BYTES_DEFAULT

    layouts = [T.Q2_0_G128, T.T3_5PB_G128]
    mats = [(layout, n, k) for layout in layouts for (n, k) in LAYER_SET] + [(T.T3_5PB_G128,) + LM_HEAD]
    set_bytes = sum(algorithmic_bytes(l, n, k, 1) for (l, n, k) in mats)
    weight_bytes = sum(n * T.row_bytes(l, k) + n * (k // GROUP) * 2 for (l, n, k) in mats)
    copies = max(2, math.ceil(3 * l2 / weight_bytes))

    # weights: `copies` independent copies of every matrix (distinct memory, same distribution)
    W = [[make_weights(torch, T, n, k, l, 1000 * c + 10 * i + rank, dev) for i, (l, n, k) in enumerate(mats)]
         for c in range(copies)]
    xs = [torch.randn((1, k), device=dev).to(torch.float16) for (_, _, k) in mats]
    ys = [torch.empty((1, n), dtype=torch.float16, device=dev) for (_, n, _) in mats]
    wss = [[T.gemv_workspace(W[c][i], 1) for i in range(len(mats))] for c in range(copies)]
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)
    launches_per_step = len(mats)

    def step(c):
        for i in range(len(mats)):
            T.gemv(W[c][i], xs[i], y=ys[i], workspace=wss[c][i], static_weights=True)

    # one CUDA graph per weight copy holds the six launches of a step
    graphs = []
    with torch.cuda.stream(stream):
        for c in range(copies):
            step(c)  # warm (sets kernel attributes outside capture)
        torch.cuda.synchronize()
        for c in range(copies):
            gph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gph, stream=stream):
                step(c)
            graphs.append(gph)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    def run_step(i):
        if args.eager:
            step(i % copies)
        else:
            graphs[i % copies].replay()

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            run_step(i)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    pci = None
    if hasattr(props, "pci_bus_id"):
        pci = f"{getattr(props, 'pci_domain_id', 0):08X}:{props.pci_bus_id:02X}:{getattr(props, 'pci_device_id', 0):02X}.0"
    with ClockSampler(local_rank, pci) as clk:
        clk.begin()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(args.steps):
                run_step(i)
            e1.record(stream)
            clk.sample_now()  # one sample while the queued replays run, however short the region
        e1.synchronize()
        clk.end()
    barrier()
    ms = e0.elapsed_time(e1)
    ms = max_over_ranks(torch, ms, world, dev)
    ms_per_step = ms / args.steps
    value = replica_throughput(set_bytes, args.steps, world, ms)

    # per-kernel launch durations in the same steady state (events around single-kernel graphs)
    per_kernel = time_kernels(torch, T, W, xs, ys, wss, mats, copies, stream)
    dom = max(per_kernel, key=lambda r: r["ms_total"])
    achieved = dom["bytes"] / (dom["ms_avg"] * 1e-3) / 1e9
    traffic = profiled_traffic(dom["key"])
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                "kernel": dom["key"], "peak_source": peaks["source"] + " hbm_gbs (copy, burst)",
                "per_kernel": [{k: (round(v, 5) if isinstance(v, float) else v) for k, v in r.items()}
                               for r in per_kernel]}

    e2e = measure_e2e(torch, T, W, mats, copies, args, stream, world, dev, set_bytes)
    # the other rows are single-GPU measurements: taken at N = 1 only, so scaling runs stay short
    extras = {} if (args.no_extras or world > 1) else measure_extras(torch, T, dev, peaks, stream)
    cpu = cpu_baseline(torch, T, W, xs, mats) if (rank == 0 and world == 1) else None

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f16 (ternary codes, fp32 accumulate)",
                "data": "synthetic (seeded codes P(0)=0.4, scales |N(0,1)|*0.02 fp16, x N(0,1) fp16)",
                "config": {"workload": WORKLOAD, "batch": 1, "layouts": ["Q2_0_g128", "T3_5PB_g128"],
                           "gemvs": [f"{'q2' if l == T.Q2_0_G128 else 't3'}_{n}x{k}" for (l, n, k) in mats],
                           "gemvs_per_step": launches_per_step, "bytes_per_step": set_bytes,
                           "l2": f"rotating {copies} weight copies ({copies * weight_bytes / 1e6:.0f} MB > 3x L2 "
                                 f"{l2 / 1e6:.0f} MB)", "parallelism": f"replicas x{world}",
                           "hbm_frac_of_8TBps": round(value / world / 8000.0, 4),
                           "launch": "tern_gemv_ex with TERN_GEMV_STATIC_WEIGHTS (programmatic dependent launch: "
                                     "each GEMV starts streaming its weights while the previous one finishes)",
                           "step_launch": "eager launches" if args.eager else "one CUDA graph replay per step"},
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches_per_step * args.steps, "clocks": clk.summary()}
        if extras:
            line["rows"] = extras
        print(json.dumps(line), flush=True)


def init_dist(world, local_rank, backend="nccl"):
    """One process per GPU (nccl), or per CPU rank (gloo, for the host-side tests of this path); ranks
    that wait for one another end with an error after two minutes."""
    import datetime
    import torch
    if backend == "nccl":
        torch.cuda.set_device(local_rank)
    torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def replica_throughput(bytes_per_step, steps, world, ms):
    """Whole-job GB/s of `world` replicas that each ran `steps` steps, timed as the max over ranks."""
    return bytes_per_step * steps * world / (ms * 1e-3) / 1e9


def max_over_ranks(torch, v, world, dev):
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def time_kernels(torch, T, W, xs, ys, wss, mats, copies, stream, reps=40):
    """Average device time per launch of each GEMV, replaying a graph of `reps` launches that rotates
    over the weight copies (HBM-cold weights), timed with CUDA events on the launching stream."""
    out = []
    for i, (layout, n, k) in enumerate(mats):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for r in range(reps):
                    c = r % copies
                    T.gemv(W[c][i], xs[i], y=ys[i], workspace=wss[c][i], static_weights=True)
            g.replay()
            torch.cuda.synchronize()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(5):
                g.replay()
            b.record(stream)
        b.synchronize()
        ms = a.elapsed_time(b) / (5 * reps)
        nb = algorithmic_bytes(layout, n, k, 1)
        out.append({"key": f"gemv_{'q2' if layout == T.Q2_0_G128 else 't3'}_{n}x{k}_b1", "bytes": nb,
                    "ms_avg": ms, "gbs": nb / (ms * 1e-3) / 1e9, "ms_total": ms})
    return out


def measure_e2e(torch, T, W, mats, copies, args, stream, world, dev, set_bytes):
    """Same step through the public C ABI with host-resident activations: per step one H2D copy of
    the step's six activation vectors from pinned memory, the six tern_gemv_ex calls, one D2H copy of
    the six results to pinned memory; all inside the event-timed region. The call arguments are
    marshalled once (ctypes), as a caller that issues the same GEMVs every decode step would."""
    lib = T.lib()
    ks = [k for (_, _, k) in mats]
    ns = [n for (_, n, _) in mats]
    hx = torch.randn((sum(ks),)).to(torch.float16).pin_memory()
    hy = torch.empty((sum(ns),), dtype=torch.float16).pin_memory()
    dx = torch.empty((sum(ks),), dtype=torch.float16, device=dev)
    dy = torch.empty((sum(ns),), dtype=torch.float16, device=dev)
    xo = [sum(ks[:i]) for i in range(len(mats))]
    yo = [sum(ns[:i]) for i in range(len(mats))]
    wss = [[T.gemv_workspace(W[c][i], 1) for i in range(len(mats))] for c in range(copies)]
    sh = ctypes.c_void_p(stream.cuda_stream)
    calls = []
    for c in range(copies):
        row = []
        for i in range(len(mats)):
            mc = W[c][i].c()
            ws = wss[c][i]
            row.append((mc, ctypes.byref(mc), ctypes.c_void_p(dx.data_ptr() + 2 * xo[i]),
                        ctypes.c_void_p(dy.data_ptr() + 2 * yo[i]),
                        ctypes.c_void_p(ws.data_ptr() if ws is not None else 0), ws.numel() if ws is not None else 0))
        calls.append(row)
    steps = max(1, min(args.steps, 500))
    bad = [0]

    def one(c):
        dx.copy_(hx, non_blocking=True)
        for (_, mref, xp, yp, wp, wn) in calls[c]:
            bad[0] |= lib.tern_gemv_ex(mref, xp, 1, yp, wp, wn, T.GEMV_STATIC_WEIGHTS, sh)
        hy.copy_(dy, non_blocking=True)

    with torch.cuda.stream(stream):
        for i in range(min(10, steps)):
            one(i % copies)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(steps):
            one(i % copies)
        b.record(stream)
    b.synchronize()
    if bad[0]:
        raise RuntimeError("tern_gemv_ex failed in the end-to-end loop")
    ms = max_over_ranks(torch, a.elapsed_time(b), world, dev)
    h2d = hx.numel() * 2
    d2h = hy.numel() * 2
    return {"value": round(set_bytes * steps * world / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 6),
            "path": "C ABI tern_gemv_ex (TERN_GEMV_STATIC_WEIGHTS) via ctypes, eager launches; one pinned H2D "
                    "of the step's activation vectors and one D2H of its results per step"}


def measure_extras(torch, T, dev, peaks, stream):
    """One line per other row of the hot path: pack, LM head, 27B batched GEMV, prefill GEMM."""
    res = {}
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def timed(fn, reps):
        # reps back-to-back calls captured in one CUDA graph; device time of a replay / reps (host
        # launch overhead of the Python binding stays out of the figure)
        with torch.cuda.stream(stream):
            fn()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _ in range(reps):
                    fn()
            g.replay()
            torch.cuda.synchronize()
            a, b = ev(), ev()
            a.record(stream)
            g.replay()
            b.record(stream)
        b.synchronize()
        del g
        return a.elapsed_time(b) / reps

    # ternarize (binarize) + pack of fp16 latents, 8B shapes (every layout)
    for layout, name in ((T.Q2_0_G128, "q2"), (T.T3_5PB_G128, "t3"), (T.Q1_0_G128, "q1")):
        tot_b, tot_ms = 0, 0.0
        for (n, k) in LAYER_SET:
            w = torch.randn((n, k), device=dev).mul_(0.02).to(torch.float16)
            s = (torch.randn((n, k // GROUP), device=dev).abs() * 0.02).to(torch.float16)
            Wp = T.pack(w, s, layout)
            ms = timed(lambda: T.pack(w, s, layout, out=Wp), 20)
            tot_b += n * k * 2 + n * (k // GROUP) * 2 + n * T.row_bytes(layout, k)
            tot_ms += ms
            del w, s, Wp
        gbs = tot_b / (tot_ms * 1e-3) / 1e9
        res[f"pack_{name}_8b_set"] = {"GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                                      "ms": round(tot_ms, 5)}

    # LM head (base-3) and 27B batched GEMVs; weights larger than L2, re-read each launch
    cases = [("lm_head_t3", T.T3_5PB_G128, 151936, 4096, b) for b in (1, 8)]
    # the binary layout on the 8B shapes: batch 1-2 is one register-kernel launch, 3-4 two, 5 and up the GEMM
    for (n, k) in LAYER_SET:
        for b in (1, 2, 4, 16):
            cases.append((f"8b_q1_{n}x{k}", T.Q1_0_G128, n, k, b))
    for layout, lname in ((T.Q2_0_G128, "q2"), (T.T3_5PB_G128, "t3")):
        for (n, k) in ((34816, 5120), (5120, 17408)):
            for b in (1, 4, 16, 64):
                cases.append((f"27b_{lname}_{n}x{k}", layout, n, k, b))
    cache = {}
    for name, layout, n, k, b in cases:
        key = (layout, n, k)
        if key not in cache:
            cache.clear()
            torch.cuda.empty_cache()
            # enough weight copies that one pass over them is over twice the 126 MB L2
            wbytes = n * T.row_bytes(layout, k) + n * (k // GROUP) * 2
            copies = max(2, min(64, -(-300_000_000 // wbytes)))
            cache[key] = [make_weights(torch, T, n, k, layout, 77 + c, dev) for c in range(copies)]
        Ws = cache[key]
        x = torch.randn((b, k), device=dev).to(torch.float16)
        y = torch.empty((b, n), dtype=torch.float16, device=dev)
        wss = [T.gemv_workspace(Wc, b) for Wc in Ws]
        it = [0]

        def f():
            c = it[0] % len(Ws)
            it[0] += 1
            T.gemv(Ws[c], x, y=y, workspace=wss[c], static_weights=True)
        ms = timed(f, 20)
        nb = algorithmic_bytes(layout, n, k, b)
        flops = 2.0 * n * k * b
        res[f"{name}_b{b}"] = {"GB/s": round(nb / (ms * 1e-3) / 1e9, 1),
                               "frac_hbm": round(nb / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                               "TFLOP/s": round(flops / (ms * 1e-3) / 1e12, 2), "us": round(ms * 1e3, 2)}
    cache.clear()
    torch.cuda.empty_cache()

    # transposed product dx = W^T dy (STE backward) on the 8B shapes, batch 1; weight copies past L2
    for layout, lname in ((T.Q2_0_G128, "q2"), (T.T3_5PB_G128, "t3"), (T.Q1_0_G128, "q1")):
        for (n, k) in ((24576, 4096), (4096, 12288)):
            wbytes = n * T.row_bytes(layout, k) + n * (k // GROUP) * 2
            copies = max(2, min(64, -(-300_000_000 // wbytes)))
            Wts = [make_weights(torch, T, n, k, layout, 6 + c, dev) for c in range(copies)]
            dy = torch.randn((1, n), device=dev).to(torch.float16)
            dxo = torch.empty((1, k), dtype=torch.float16, device=dev)
            nbw = int(T.lib().tern_gemv_t_workspace_bytes(ctypes.byref(Wts[0].c()), 1))
            wsv = torch.empty(max(nbw, 16), dtype=torch.uint8, device=dev)
            it = [0]

            def ft():
                c = it[0] % len(Wts)
                it[0] += 1
                T.gemv_t(Wts[c], dy, dx=dxo, workspace=wsv if nbw else None)
            ms = timed(ft, 20)
            nb = algorithmic_bytes(layout, n, k, 1)
            res[f"gemv_t_{lname}_{n}x{k}_b1"] = {"GB/s": round(nb / (ms * 1e-3) / 1e9, 1),
                                                 "frac_hbm": round(nb / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                                                 "us": round(ms * 1e3, 2),
                                                 "note": f"{copies} weight copies (HBM-cold); partials "
                                                         f"{nbw / 1e6:.1f} MB written and re-read"}
            del Wts
            torch.cuda.empty_cache()

    # activation-side block Hadamard rotation (sign flip + FWHT per 1024-block) in front of a GEMV
    signs = torch.where(torch.rand(1024, device=dev) < 0.5, -1, 1).to(torch.int8)
    for b, k in ((1, 4096), (1, 12288), (64, 17408)):
        xr = torch.randn((b, k), device=dev).to(torch.float16)
        yr = torch.empty_like(xr)
        ms = timed(lambda: T.hadamard_rotate(xr, signs, y=yr), 50)
        nb = 2 * (2 * b * k) + 1024
        res[f"rotate_b{b}_k{k}"] = {"us": round(ms * 1e3, 2), "GB/s": round(nb / (ms * 1e-3) / 1e9, 1),
                                    "note": "latency-bound (a few KB per call)" if b == 1 else "HBM"}

    # prefill GEMM M=2048, K=5120, N=17408 on tcgen05, both layouts (the prefill config is Q2_0_g128;
    # the base-3 line is the same product on the denser layout)
    M, N, K = 2048, 17408, 5120
    X = torch.randn((M, K), device=dev).to(torch.float16)
    Y = torch.empty((M, N), dtype=torch.float16, device=dev)
    for layout, lname in ((T.Q2_0_G128, "q2"), (T.T3_5PB_G128, "t3"), (T.Q1_0_G128, "q1")):
        key = f"gemm_{lname}_2048x17408x5120"
        try:
            Wg = make_weights(torch, T, N, K, layout, 5, dev)
            ms = timed(lambda: T.gemm(Wg, X, Y=Y), 20)
            tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
            res[key] = {"TFLOP/s": round(tf, 1), "frac_fp16_peak": round(tf / peaks["bf16_tflops"], 4),
                        "peak_TFLOP/s": peaks["bf16_tflops"], "ms": round(ms, 4)}
            del Wg
        except Exception as e:  # the GEMM is reported, not required for the GEMV metric
            res[key] = {"error": str(e)[:200]}
    return res


def host_cpu():
    """(logical CPUs, model name) of the host, as `nproc` and `lscpu` report them."""
    n = os.cpu_count() or 1
    model = None
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.lower().startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except Exception:
        pass
    if model is None:
        try:
            with open("/proc/cpuinfo") as f:
                for line in f:
                    if line.startswith("model name"):
                        model = line.split(":", 1)[1].strip()
                        break
        except Exception:
            model = "unknown"
    return n, model


def cpu_baseline(torch, T, W, xs, mats, rows=1024, seconds=8.0):
    """The oracle, as it stands, on a bounded sample (`rows` rows of each GEMV of the step), timed on
    one thread and on all of the host's cores (numpy's BLAS threads); the all-cores figure is the
    reported value."""
    import numpy as np
    import oracle as O
    try:
        from threadpoolctl import threadpool_limits
    except Exception:  # pragma: no cover
        threadpool_limits = None
    samples = []
    nbytes = 0
    for i, (layout, n, k) in enumerate(mats):
        Wm = W[0][i]
        r = np.arange(min(rows, n))
        codes = Wm.codes[: len(r)].cpu().numpy()
        sc = Wm.scales[: len(r), : k // GROUP].cpu().numpy()
        x = xs[i].cpu().numpy()
        samples.append((codes, sc, x, layout, k))
        nbytes += algorithmic_bytes(layout, len(r), k, 1)

    def leg(threads):
        ctx = threadpool_limits(limits=threads) if threadpool_limits else None
        t0 = time.perf_counter()
        reps = 0
        while True:
            for (codes, sc, x, layout, k) in samples:
                O.gemv(codes, sc, x, layout, k)
            reps += 1
            if time.perf_counter() - t0 > seconds or reps >= 50:
                break
        dt = time.perf_counter() - t0
        if ctx is not None and hasattr(ctx, "unregister"):
            ctx.unregister()
        return nbytes * reps / dt / 1e9, reps, dt

    ncpu, model = host_cpu()
    v1, r1, d1 = leg(1)
    va, ra, da = leg(ncpu)
    return {"value": round(va, 4), "unit": "GB/s", "cores": ncpu, "kind": "oracle",
            "sample": f"first {rows} rows of each of the {len(mats)} GEMVs of the step x {ra} passes ({da:.1f} s, "
                      f"numpy fp64, {ncpu} threads)",
            "one_thread": {"value": round(v1, 4), "unit": "GB/s", "cores": 1,
                           "sample": f"the same sample x {r1} passes ({d1:.1f} s)"},
            "host": {"nproc": ncpu, "cpu_model": model}}


def record_traffic(csv_path):
    """Writes profiles/traffic.json from an ncu --csv capture (one or more launches of the dominant
    GEMV): dram read + write bytes per launch, keyed by the digest of the kernel source it ran."""
    import csv
    rows = list(csv.reader(open(csv_path)))
    head = None
    vals = {}
    for r in rows:
        if "Metric Name" in r and "Metric Value" in r:
            head = r
            continue
        if head is None or len(r) != len(head):
            continue
        d = dict(zip(head, r))
        if d.get("Metric Name") in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            unit = d.get("Metric Unit", "byte").lower()
            scale = {"byte": 1, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9}.get(unit, 1)
            v = float(d["Metric Value"].replace(",", "")) * scale
            vals.setdefault(d.get("ID", "0"), {})[d["Metric Name"]] = v
    per = [v.get("dram__bytes_read.sum", 0) + v.get("dram__bytes_write.sum", 0) for v in vals.values()]
    if not per:
        raise SystemExit("no dram__bytes metrics in " + csv_path)
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(path))
    except Exception:
        d = {}
    key = os.environ.get("TRAFFIC_KEY", "gemv_t3_151936x4096_b1")
    d[key] = {"dram_bytes_per_launch": int(round(statistics.median(per))), "launches": len(per),
              "source": "tern_gemv_i8.cu", "source_sha": source_digest("tern_gemv_i8.cu"),
              "note": "recorded by bench.py --record-traffic from an ncu capture of this source"}
    with open(path, "w") as f:
        json.dump(d, f, indent=1)
    print(json.dumps({key: d[key]}))


# -------------------------------------------------------------------------- the reference arm
def run_reference(args, rank, world):
    """The CPU oracle timed on the host cores on a bounded sample of the same workload."""
    if rank != 0:
        return
    import numpy as np
    import oracle as O
    from gemm_tern_gemv_b200 import synth
    try:
        from threadpoolctl import threadpool_limits
        lim = threadpool_limits(limits=1)
    except Exception:
        lim = None
    rows = 256
    samples, nbytes = [], 0
    cases = [(layout, mi, n, k) for layout in (O.Q2_0_G128, O.T3_5PB_G128) for mi, (n, k) in enumerate(LAYER_SET)]
    cases.append((O.T3_5PB_G128, 3, LM_HEAD[0], LM_HEAD[1]))
    for layout, mi, n, k in cases:
        seed = synth.seed_for(2, mi) + 10 * layout
        t = synth.ternary_codes(rows, k, seed)
        s = synth.group_scales(rows, k // GROUP, seed)
        x = synth.activations(1, k, seed)
        samples.append((O.pack(t, layout), s, x, layout, k))
        nbytes += rows * O.row_bytes(layout, k) + rows * (k // GROUP) * 2 + 2 * k + 2 * rows

    def step():
        for (codes, s, x, layout, k) in samples:
            O.gemv(codes, s, x, layout, k)
    for _ in range(max(0, args.warmup)):
        step()
    steps = max(1, args.steps)
    t0 = time.perf_counter()
    done = 0
    for _ in range(steps):
        step()
        done += 1
        if time.perf_counter() - t0 > 120.0:
            break
    dt = time.perf_counter() - t0
    v = nbytes * done / dt / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
            "steps": done, "warmup": args.warmup, "ms_per_step": round(dt / done * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded, same distributions)",
            "config": {"workload": WORKLOAD, "batch": 1, "sample_rows_per_matrix": rows},
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"{rows} rows of each of the seven GEMVs per step (numpy fp64, 1 thread)"},
            "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


PROFILE_ALL = ["gemv_t3_151936x4096_b1", "gemv_q2_24576x4096_b1", "gemv_q2_34816x5120_b16", "gemm_q2_2048x17408x5120",
               "gemm_t3_2048x17408x5120", "pack_q2_24576x4096", "pack_t3_24576x4096", "pack_q1_24576x4096",
               "unpack_q2_24576x4096", "gemvt_q2_24576x4096_b1", "rotate_b64_k17408"]


def run_profile_case(case: str, launches: int = 6):
    """A handful of launches of one kernel case, for an ncu capture (no timing claims). 'all' runs
    two launches of every case in PROFILE_ALL, one kernel family after another."""
    import torch
    import gemm_tern_gemv_b200 as T
    if case == "all":
        for c in PROFILE_ALL:
            run_profile_case(c, 2)
        return
    dev = torch.device("cuda", 0)
    parts = case.split("_")
    kind = parts[0]
    layout = {"q2": T.Q2_0_G128, "t3": T.T3_5PB_G128, "q1": T.Q1_0_G128}.get(parts[1])
    if kind == "gemv":
        n, k = (int(v) for v in parts[2].split("x"))
        b = int(parts[3][1:])
        W = make_weights(torch, T, n, k, layout, 1, dev)
        x = torch.randn((b, k), device=dev).to(torch.float16)
        ws = T.gemv_workspace(W, b)
        fn = lambda: T.gemv(W, x, workspace=ws, static_weights=True)
    elif kind == "gemvt":
        n, k = (int(v) for v in parts[2].split("x"))
        b = int(parts[3][1:])
        W = make_weights(torch, T, n, k, layout, 1, dev)
        dy = torch.randn((b, n), device=dev).to(torch.float16)
        fn = lambda: T.gemv_t(W, dy)
    elif kind == "gemm":
        m, n, k = (int(v) for v in parts[2].split("x"))
        W = make_weights(torch, T, n, k, layout, 1, dev)
        X = torch.randn((m, k), device=dev).to(torch.float16)
        fn = lambda: T.gemm(W, X)
    elif kind == "pack":
        n, k = (int(v) for v in parts[2].split("x"))
        w = torch.randn((n, k), device=dev).mul_(0.02).to(torch.float16)
        s = (torch.randn((n, k // GROUP), device=dev).abs() * 0.02).to(torch.float16)
        Wp = T.pack(w, s, layout)
        fn = lambda: T.pack(w, s, layout, out=Wp)
    elif kind == "unpack":
        n, k = (int(v) for v in parts[2].split("x"))
        W = make_weights(torch, T, n, k, layout, 1, dev)
        fn = lambda: T.unpack(W, want_w=True, want_t=False)
    elif kind == "rotate":
        b, k = int(parts[1][1:]), int(parts[2][1:])
        signs = torch.where(torch.rand(1024, device=dev) < 0.5, -1, 1).to(torch.int8)
        xr = torch.randn((b, k), device=dev).to(torch.float16)
        fn = lambda: T.hadamard_rotate(xr, signs)
    else:
        raise SystemExit(f"unknown case {case}")
    for _ in range(launches):
        fn()
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": case, "launches": launches}))


def main():
    args = parse()
    if args.record_traffic:
        record_traffic(args.record_traffic)
        return
    if args.profile:
        run_profile_case(args.profile)
        return
    world = _env_int("WORLD_SIZE", 1)
    rank = _env_int("RANK", 0)
    local_rank = _env_int("LOCAL_RANK", 0)
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        init_dist(world, local_rank, "nccl")
    try:
        run_native(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
