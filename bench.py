#!/usr/bin/env python
"""Benchmark: MoE layer forward tokens/s on B200, and its roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one whole layer forward (router, aux loss, capacity dispatch + gather,
both grouped expert GEMMs, combine) over one batch of T synthetic tokens, inputs
resident in HBM.  With N > 1 (launched by torch.distributed.run) every rank runs
its own batch as its own routing group: the units are independent, there is no
data-path collective, and the scaling is weak; the job value is the tokens of
all ranks over the slowest rank's device time.

`--impl reference` times the CPU oracle (the plain definition, single-threaded
C) on the host cores on a bounded sample of the same workload.
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_sparse_b200.configs import WORKLOADS  # noqa: E402

METRIC = "MoE layer fwd tokens/s at 1 B200; % of bf16 TC/HBM roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic of the first grouped GEMM launch (dram__bytes_read.sum +
# dram__bytes_write.sum) from one ncu capture, keyed by workload, valid only
# for the kernel source it was measured on.
NCU_TRAFFIC = {
    # python bench.py --steps 3 --warmup 3 --no-cpu-baseline, then under
    # ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum --clock-control none
    #     -k regex:grouped_gemm -s 6 -c 2 (first timed step): stage 1 read
    # 402836224 B (W1 + xe, the compulsory set) and wrote 362386432 B (H, part
    # of it still in L2 when the kernel ends).  Keyed to the sources below; since
    # the capture common.cuh only gained declarations the GEMM does not use.
    "switch_base": {"bytes_per_launch": 402836224 + 362386432, "src_sha": "7340ddffc88f93d6"},
}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def gemm_source_sha():
    h = hashlib.sha256()
    for name in ("gemm_tc.cu", "common.cuh"):
        with open(os.path.join(ROOT, "mixture_experts_sparse_b200", "csrc", name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


# ------------------------------------------------------------------ events ----

class RawEvents:
    """CUDA events created and timed through the CUDA runtime directly (the
    library records them inside moe_forward_events, out of torch's sight)."""

    def __init__(self):
        import ctypes
        import glob
        import torch
        self.ct = ctypes
        lib = None
        for name in ("libcudart.so.12", "libcudart.so"):
            try:
                lib = ctypes.CDLL(name)
                break
            except OSError:
                pass
        if lib is None:
            pat = os.path.join(os.path.dirname(torch.__file__), "..", "nvidia", "cuda_runtime", "lib", "libcudart.so*")
            lib = ctypes.CDLL(sorted(glob.glob(pat))[0])
        self.lib = lib
        self.handles = []

    def create(self):
        h = self.ct.c_void_p()
        if self.lib.cudaEventCreate(self.ct.byref(h)) != 0:
            raise RuntimeError("cudaEventCreate failed")
        self.handles.append(h)
        return h

    def record(self, h, stream):
        if self.lib.cudaEventRecord(h, self.ct.c_void_p(stream.cuda_stream)) != 0:
            raise RuntimeError("cudaEventRecord failed")

    def ms(self, a, b):
        out = self.ct.c_float()
        if self.lib.cudaEventElapsedTime(self.ct.byref(out), a, b) != 0:
            raise RuntimeError("cudaEventElapsedTime failed")
        return out.value

    def close(self):
        for h in self.handles:
            self.lib.cudaEventDestroy(h)
        self.handles = []


# ------------------------------------------------------------------ clocks ----

class SmiSampler:
    """Fallback: nvidia-smi's own sampling loop (the profiling recipe's clocks line)."""
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        import subprocess
        import tempfile
        import torch
        props = torch.cuda.get_device_properties(device_index)
        self.bus = ("%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)).lower()
        self.tmp = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
        self.proc = subprocess.Popen(["nvidia-smi", "--id=" + self.bus, "--query-gpu=" + self.FIELDS,
                                      "--format=csv,noheader,nounits", "-lms", "50"],
                                     stdout=self.tmp, stderr=subprocess.DEVNULL)

    def stop(self):
        self.proc.terminate()
        self.proc.wait()
        self.tmp.seek(0)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.tmp.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 6:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[2:]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.tmp.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi -lms 50"}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x10: "sync_boost"}

    def __init__(self, device_index):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId_v2(bus.encode())
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as exc:   # noqa: BLE001
            self.ok = False
            self.error = repr(exc)
        self.smi = None
        if not self.ok:
            try:
                self.smi = SmiSampler(device_index)
            except Exception as exc:   # noqa: BLE001
                self.error = getattr(self, "error", "") + " / " + repr(exc)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.reasons |= int(r)
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self.smi is not None:
            return self.smi.stop()
        if self._thread:
            self._stop.set()
            self._thread.join()
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "error": getattr(self, "error", None)}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples), "source": "NVML, every 2 ms"}


# ------------------------------------------------------------- cpu oracle ----

def oracle_tokens_per_s(L, w, target_s, max_tokens=None):
    """Time the oracle (single-threaded C) on the first n tokens of the batch,
    treated as its own routing group; n is grown until a run takes target_s."""
    import oracle
    W = {k: L[k] for k in ("w1", "b1", "w3", "b3", "w2", "b2")}
    act = oracle.SWIGLU if w.act == "swiglu" else oracle.RELU
    out_dtype = oracle.BF16 if w.dtype == "bf16" else oracle.F32
    limit = max_tokens or w.T

    def run(n):
        C = oracle.capacity(n, w.n_experts, w.top_k, w.capacity_factor)
        t0 = time.perf_counter()
        oracle.forward(L["x"][:n], L["w_r"], L["b_r"], W, k=w.top_k, C=C, act=act, alpha=w.alpha,
                       out_dtype=out_dtype)
        return time.perf_counter() - t0

    # start where every expert has a few slots, so the probe does expert work
    n = int(min(limit, max(64, -(-16 * w.n_experts // max(1, int(w.top_k * w.capacity_factor))))))
    dt = run(n)
    for _ in range(4):   # a few probes, each aiming slightly past the target
        if dt >= target_s or n >= limit:
            break
        n = int(min(limit, 4 * n, max(2 * n if dt < 0.25 * target_s else n + 1,
                                      n * 1.15 * target_s / max(dt, 1e-6))))
        dt = run(n)
    return n / dt, n, dt


# ------------------------------------------------------------- multi-rank ----

def max_over_ranks(local_ms, world, device="cuda"):
    """Slowest rank's time: every rank contributes its own device time."""
    if world == 1:
        return float(local_ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank, world, steps, max_ms):
    """Whole-job throughput: the tokens of all ranks over the slowest rank's time
    (each rank runs its own batch as its own routing group: weak scaling)."""
    return tokens_per_rank * world * steps / (max_ms * 1e-3)


# ------------------------------------------------------------------ main ----

def layer_work(w, kept_rows, touched):
    """Algorithmic FLOPs and bytes of one layer forward (kept assignments only)."""
    d, dff = w.d_model, w.d_ff
    esz = 2 if w.dtype == "bf16" else 4
    g1 = (4 if w.act == "swiglu" else 2) * d * dff * kept_rows
    g2 = 2 * d * dff * kept_rows
    per_expert_w = (3 if w.act == "swiglu" else 2) * d * dff * esz
    bytes_alg = 2 * w.T * d * esz + touched * per_expert_w + w.n_experts * d * 4
    return g1, g2, bytes_alg


def run_ours(args, rank, world, local):
    import numpy as np
    import torch
    import torch.distributed as dist

    from mixture_experts_sparse_b200 import inputs
    from mixture_experts_sparse_b200 import native as nat
    from mixture_experts_sparse_b200.layer import MoeLayer, to_device

    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    w = WORKLOADS[args.workload]
    if args.tokens:
        w = w.scaled(T=args.tokens)
    C = nat.moe_capacity(w.T, w.n_experts, w.top_k, w.capacity_factor)
    L = inputs.make_workload(w, seed=w.seed + rank)
    layer = MoeLayer(w.T, w.d_model, w.d_ff, w.n_experts, w.top_k, C, w.dtype, w.act, L, alpha=w.alpha)
    x = to_device(L["x"])
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        nat.check(layer.forward(x, routing_outputs=False))
    torch.cuda.synchronize()
    nat.check(nat.moe_read_device_status(layer.ws))

    # ---- device-timed region: K forwards, stage events recorded inside --------
    K = args.steps
    rev = RawEvents()
    ev = [[rev.create() for _ in range(6)] for _ in range(K)]
    start, stop = rev.create(), rev.create()
    sampler = ClockSampler(local)
    w_ = layer.w
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    rev.record(start, stream)
    for i in range(K):
        nat.check(nat.moe_forward_events(layer.cfg, x, w_["w_r"], w_["b_r"], w_["w1"], w_["b1"], w_["w3"],
                                         w_["b3"], w_["w2"], w_["b2"], layer.out, offsets=layer.offsets,
                                         kept=layer.kept, aux=layer.aux, ws=layer.ws, events=ev[i]))
    rev.record(stop, stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    nat.check(nat.moe_read_device_status(layer.ws))
    t_ms = max_over_ranks(rev.ms(start, stop), world)
    # ---- the same forward replayed from a CUDA graph (one launch per step) ------
    graph_ms = None
    if not args.no_graph:
        g = torch.cuda.CUDAGraph()
        s_cap = torch.cuda.Stream()
        s_cap.wait_stream(stream)
        with torch.cuda.stream(s_cap):
            nat.check(layer.forward(x, routing_outputs=False))
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s_cap):
            nat.check(layer.forward(x, routing_outputs=False))
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        barrier()
        sampler_g = ClockSampler(local)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sampler_g.start()
        g0.record(stream)
        for _ in range(K):
            g.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        barrier()
        clocks = sampler_g.stop()
        nat.check(nat.moe_read_device_status(layer.ws))
        graph_ms = max_over_ranks(g0.elapsed_time(g1), world)
        del g
    main_ms = graph_ms if graph_ms is not None else t_ms

    stage = np.array([[rev.ms(ev[i][j], ev[i][j + 1]) for j in range(5)] for i in range(K)])
    stage_ms = stage.mean(axis=0)
    rev.close()
    kept_rows = int(layer.offsets[-1].item())
    touched = int((layer.kept > 0).sum().item())

    # ---- end to end: host input -> device -> forward -> host output -----------
    # Every step copies its input from pinned host memory and its output (and
    # aux loss) back.  The copies of neighbouring steps overlap the forward on
    # their own streams (double-buffered device input and output; the forward
    # itself stays on one stream, so the workspace is never shared in flight).
    xh = torch.empty(x.shape, dtype=x.dtype).pin_memory()
    xh.copy_(x.cpu())
    oh = [torch.empty(layer.out.shape, dtype=layer.out.dtype).pin_memory() for _ in range(2)]
    ah = [torch.empty(1, dtype=torch.float64).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(x) for _ in range(2)]
    od = [torch.empty_like(layer.out) for _ in range(2)]
    auxd = [torch.empty(1, dtype=torch.float64, device="cuda") for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]      # input slot filled
    ev_done = [torch.cuda.Event() for _ in range(2)]    # forward of the slot finished
    ev_out = [torch.cuda.Event() for _ in range(2)]     # output slot copied out
    wl = layer.w

    def e2e_step(i):
        j = i & 1
        if i >= 2:
            s_in.wait_event(ev_done[j])                 # forward i-2 has read xd[j]
        with torch.cuda.stream(s_in):
            xd[j].copy_(xh, non_blocking=True)
            ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        if i >= 2:
            stream.wait_event(ev_out[j])                # od[j] of step i-2 is on the host
        nat.check(nat.moe_forward(layer.cfg, xd[j], wl["w_r"], wl["b_r"], wl["w1"], wl["b1"], wl["w3"], wl["b3"],
                                  wl["w2"], wl["b2"], od[j], aux=auxd[j], ws=layer.ws, stream=stream))
        ev_done[j].record(stream)
        s_out.wait_event(ev_done[j])
        with torch.cuda.stream(s_out):
            oh[j].copy_(od[j], non_blocking=True)
            ah[j].copy_(auxd[j], non_blocking=True)
            ev_out[j].record(s_out)

    def e2e_run(n):
        for i in range(n):
            e2e_step(i)
        stream.wait_event(ev_out[(n - 1) & 1])
        if n >= 2:
            stream.wait_event(ev_out[(n - 2) & 1])

    e2e_run(max(3, min(args.warmup, 10)))
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    e2e_run(K)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    nat.check(nat.moe_read_device_status(layer.ws))
    h2d = x.numel() * x.element_size()
    d2h = layer.out.numel() * layer.out.element_size() + 8

    # ---- roofline --------------------------------------------------------------
    pk, pk_src = peaks()
    peak_tf = pk["bf16_tflops"]
    peak_bw = pk["hbm_gbs"]
    g1, g2, bytes_alg = layer_work(w, kept_rows, touched)
    gemm1_ms = float(stage_ms[2])
    achieved_tf = g1 / (gemm1_ms * 1e-3) / 1e12
    traffic = None
    tr = NCU_TRAFFIC.get(args.workload)
    if tr and tr.get("src_sha") == gemm_source_sha():
        traffic = tr["bytes_per_launch"]
    step_ms = main_ms / K
    layer_roof_ms = max((g1 + g2) / (peak_tf * 1e12), bytes_alg / (peak_bw * 1e9)) * 1e3

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, n, dt = oracle_tokens_per_s(L, w, args.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"first {n} tokens of the batch as one routing group (C from the same cf), "
                         f"full layer forward in the single-threaded C oracle, {dt:.1f} s"}

    launches_per_step = 6 + (0 if (w.dtype == "bf16" and w.top_k == 1) else 1)
    if rank == 0:
        line = {
            "metric": METRIC, "value": job_tokens_per_s(w.T, world, K, main_ms), "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "T": w.T, "d_model": w.d_model, "d_ff": w.d_ff,
                       "n_experts": w.n_experts, "top_k": w.top_k, "capacity_factor": w.capacity_factor,
                       "capacity": C, "act": w.act, "router": "fp32",
                       "l2": "inputs larger than L2: x + expert weights = %.0f MB > 126 MB, no flush"
                             % ((w.T * w.d_model * 2 + w.n_experts * (3 if w.act == 'swiglu' else 2)
                                 * w.d_model * w.d_ff * 2) / 1e6),
                       "parallelism": "replicas (one routing group per GPU)" if world > 1 else "single GPU",
                       "launch": "CUDA graph replay of moe_forward" if graph_ms is not None else "moe_forward calls",
                       "eager_ms_per_step": t_ms / K,
                       "kept_assignments": kept_rows, "touched_experts": touched},
            "roofline": {"bound": "tensor", "kernel": "grouped_gemm stage 1 (x W1^T + act)",
                         "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": achieved_tf / peak_tf, "traffic": traffic,
                         "peak_source": f"{pk_src} bf16 burst (MEASURED_PEAKS.json bf16_tflops)",
                         "flops_per_launch": g1, "avg_launch_ms": gemm1_ms},
            "layer_roofline": {"flops": g1 + g2, "bytes": bytes_alg, "roofline_ms": layer_roof_ms,
                               "frac": layer_roof_ms / step_ms},
            "stages_ms": {"router+aux": stage_ms[0], "dispatch+gather": stage_ms[1], "gemm1": stage_ms[2],
                          "gemm2": stage_ms[3], "combine": stage_ms[4]},
            "cpu_baseline": cpu,
            "e2e": {"value": job_tokens_per_s(w.T, world, K, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / K,
                    "overlap": "copies of neighbouring steps overlap the forward (two copy streams)"},
            "gpu_launches": launches_per_step * K,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_reference(args, rank, world):
    if rank != 0:
        return
    import numpy as np  # noqa: F401
    from mixture_experts_sparse_b200 import inputs
    from oracle import capacity

    w = WORKLOADS[args.workload]
    if args.tokens:
        w = w.scaled(T=args.tokens)
    L = inputs.make_workload(w)
    C = capacity(w.T, w.n_experts, w.top_k, w.capacity_factor)
    # size one step so the whole run stays within a few minutes
    per_step = max(0.5, min(6.0, args.reference_budget_s / (args.steps + args.warmup)))
    _, n, dt = oracle_tokens_per_s(L, w, per_step)
    import oracle
    Wt = {k: L[k] for k in ("w1", "b1", "w3", "b3", "w2", "b2")}
    act = oracle.SWIGLU if w.act == "swiglu" else oracle.RELU
    out_dtype = oracle.BF16 if w.dtype == "bf16" else oracle.F32
    Cn = oracle.capacity(n, w.n_experts, w.top_k, w.capacity_factor)

    def step():
        oracle.forward(L["x"][:n], L["w_r"], L["b_r"], Wt, k=w.top_k, C=Cn, act=act, alpha=w.alpha,
                       out_dtype=out_dtype)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    v = n * args.steps / el
    line = {
        "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": w.name, "T": w.T, "d_model": w.d_model, "d_ff": w.d_ff, "n_experts": w.n_experts,
                   "top_k": w.top_k, "capacity_factor": w.capacity_factor, "capacity": C, "act": w.act},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"each step: the first {n} tokens of the batch as one routing group, full "
                                   f"layer forward in the single-threaded C oracle"},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="switch_base")
    ap.add_argument("--tokens", type=int, default=None, help="override the workload's T (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time direct moe_forward calls instead of graph replay")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--reference-budget-s", type=float, default=150.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and world == 1 and args.gpus > 1:
        ap.error("--gpus N > 1 runs under torch.distributed.run (one process per GPU)")
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
