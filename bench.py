#!/usr/bin/env python
"""Benchmark: MoE layer forward tokens/s on B200, and its roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one whole layer forward (router, aux loss, capacity dispatch + gather,
both grouped expert GEMMs, combine) over one batch of T synthetic tokens, inputs
resident in HBM.  The JSON line's headline is the Switch-Base workload; its
"workloads" block times every synthetic workload (Switch-Base, top-2, skew,
Mixtral, tiny fp32) the same way, each with its layer roofline fraction, its
dominant kernel's fraction and the SM clocks seen while it ran.

With N > 1 (launched by torch.distributed.run) the N ranks hold the shards of
ONE routing group of N x T tokens (T per rank: weak scaling): each rank routes
its own tokens, the ranks all-gather their per-expert claim counts (the one
exchange slot claiming in token order needs), and every rank then dispatches,
runs the experts and combines its own tokens -- the result is the single-GPU
forward of the whole group.  `--replicas` instead runs one independent routing
group per GPU with no data-path collective.

`--impl reference` times the CPU oracle (the plain definition, C, fp64) on the
host cores on a bounded sample of the same workload.
"""
import argparse
import concurrent.futures
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

from mixture_experts_sparse_b200.configs import ORDER, WORKLOADS  # noqa: E402

METRIC = "MoE layer fwd tokens/s at 1 B200; % of bf16 TC/HBM roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP32_PEAK_NOTE = "148 SMs x 128 FP32 lanes x 2 flop x SM clock"

# DRAM traffic of the first grouped GEMM launch (dram__bytes_read.sum +
# dram__bytes_write.sum) from one ncu capture, keyed by workload, valid only
# for the kernel source it was measured on.
NCU_TRAFFIC = {
    # python bench.py --only --steps 3 --warmup 3 --no-cpu-baseline --no-backward --workload switch_base,
    # then the same under ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum --clock-control none
    #     -k regex:grouped_gemm -s 6 -c 2 (first timed forward): stage 1 read 402801664 B (W1 + xe, the
    # compulsory set) and wrote 361353728 B (H, part of it still in L2 when the kernel ends).  Keyed to the
    # GEMM's sources (gemm_tc.cu, tc_common.cuh) at the capture.
    "switch_base": {"bytes_per_launch": 402801664 + 361353728, "src_sha": "b39b3c9c3aa50846"},
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
    for name in ("gemm_tc.cu", "tc_common.cuh"):
        with open(os.path.join(ROOT, "mixture_experts_sparse_b200", "csrc", name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def host_threads():
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1))


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
                                      "--format=csv,noheader,nounits", "-lms", "20"],
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
                "samples": len(sm), "source": "nvidia-smi -lms 20"}


def nvml_handle(device_index):
    """NVML handle of torch's device `device_index`: by PCI bus id (both hex
    cases), then by UUID, then by index.  Returns (pynvml, handle, how) or
    raises with every attempt's error."""
    import pynvml
    import torch
    pynvml.nvmlInit()
    props = torch.cuda.get_device_properties(device_index)
    errs = []
    bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
    for b in (bus.upper(), bus):
        for fn in ("nvmlDeviceGetHandleByPciBusId_v2", "nvmlDeviceGetHandleByPciBusId"):
            try:
                return pynvml, getattr(pynvml, fn)(b.encode() if fn.endswith("_v2") else b), "pci " + b
            except Exception as exc:   # noqa: BLE001
                errs.append(f"{fn}({b}): {exc!r}")
    uid = getattr(props, "uuid", None)
    if uid is not None:
        u = str(uid)
        u = u if u.startswith("GPU-") else "GPU-" + u
        try:
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(u), "uuid"
        except Exception as exc:   # noqa: BLE001
            errs.append(f"uuid {u}: {exc!r}")
    if not os.environ.get("CUDA_VISIBLE_DEVICES"):
        try:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(device_index), "index"
        except Exception as exc:   # noqa: BLE001
            errs.append(f"index: {exc!r}")
    raise RuntimeError("; ".join(errs))


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (every 1 ms) while
    running; falls back to nvidia-smi's sampling loop."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x10: "sync_boost"}

    def __init__(self, device_index):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        self.error = None
        try:
            self.nv, self.h, self.how = nvml_handle(device_index)
            self.max_mhz = self.nv.nvmlDeviceGetMaxClockInfo(self.h, self.nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception as exc:   # noqa: BLE001
            self.error = repr(exc)[:600]
        self.smi = None
        if not self.ok:
            try:
                self.smi = SmiSampler(device_index)
            except Exception as exc:   # noqa: BLE001
                self.error = (self.error or "") + " / " + repr(exc)

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
            except Exception:   # noqa: BLE001
                pass
            time.sleep(0.001)

    def start(self):
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self.smi is not None:
            out = self.smi.stop()
            out["nvml_error"] = self.error
            return out
        if self._thread:
            self._stop.set()
            self._thread.join()
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "error": self.error}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples), "source": f"NVML every 1 ms ({self.how})"}


# ------------------------------------------------------------- cpu oracle ----

def oracle_forward_seconds(L, w, n, threads):
    """Wall time of the oracle's whole layer forward over the first n tokens of
    the batch as one routing group: routing, aux loss and the serial slot claim
    once, then the per-token expert work (the oracle's single-threaded per-token
    function) over `threads` host threads, one token chunk per task."""
    import numpy as np

    import oracle
    W = {k: L[k] for k in ("w1", "b1", "w3", "b3", "w2", "b2")}
    act = oracle.SWIGLU if w.act == "swiglu" else oracle.RELU
    out_dtype = oracle.BF16 if w.dtype == "bf16" else oracle.F32
    x = L["x"][:n]
    C = oracle.capacity(n, w.n_experts, w.top_k, w.capacity_factor)
    t0 = time.perf_counter()
    if threads <= 1:
        oracle.forward(x, L["w_r"], L["b_r"], W, k=w.top_k, C=C, act=act, alpha=w.alpha, out_dtype=out_dtype)
        return time.perf_counter() - t0
    routing = oracle.route(x, L["w_r"], L["b_r"], w.top_k)
    oracle.aux_loss(routing["idx"], routing["probs"], w.alpha)
    disp = oracle.dispatch(routing["idx"], w.n_experts, C)
    chunk = max(1, -(-n // (4 * threads)))
    parts = [np.arange(i, min(n, i + chunk), dtype=np.int64) for i in range(0, n, chunk)]
    with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(lambda tk: oracle.layer_tokens(x, W, routing, disp, tk, act, out_dtype), parts))
    return time.perf_counter() - t0


def oracle_tokens_per_s(L, w, target_s, threads=1, max_tokens=None):
    """Oracle throughput on the first n tokens of the batch, n grown until one
    run takes about target_s.  Returns (tokens/s, n, seconds)."""
    limit = max_tokens or w.T
    n = int(min(limit, max(64 * threads, -(-16 * w.n_experts // max(1, int(w.top_k * w.capacity_factor))))))
    dt = oracle_forward_seconds(L, w, n, threads)
    for _ in range(5):   # a few probes, each aiming slightly past the target
        if dt >= target_s or n >= limit:
            break
        n = int(min(limit, 4 * n, max(2 * n if dt < 0.25 * target_s else n + 1,
                                      n * 1.15 * target_s / max(dt, 1e-6))))
        dt = oracle_forward_seconds(L, w, n, threads)
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
    """Whole-job throughput: the tokens of all ranks over the slowest rank's time."""
    return tokens_per_rank * world * steps / (max_ms * 1e-3)


# ------------------------------------------------------------------ work ----

def layer_work(w, kept_rows, touched, T=None):
    """Algorithmic FLOPs of the two expert GEMMs and compulsory bytes of one
    layer forward (kept assignments only; x + out + touched expert weights + W_r)."""
    T = w.T if T is None else T
    d, dff = w.d_model, w.d_ff
    esz = 2 if w.dtype == "bf16" else 4
    g1 = (4 if w.act == "swiglu" else 2) * d * dff * kept_rows
    g2 = 2 * d * dff * kept_rows
    per_expert_w = (3 if w.act == "swiglu" else 2) * d * dff * esz
    bytes_alg = 2 * T * d * esz + touched * per_expert_w + w.n_experts * d * 4
    return g1, g2, bytes_alg


def stage_roofline(stage, w, kept_rows, touched, ms, pk):
    """Roofline of one stage of the forward from its event-timed duration.
    gemm1/gemm2: tensor-bound, algorithmic FLOPs of the kept rows; router:
    HBM, one read of x + W_r + the routing outputs; dispatch+gather: HBM,
    idx/gate in, pos/drop/row maps out, x rows read and written for kept
    assignments, output rows zeroed for fully dropped tokens (top-1 fused);
    combine: HBM, k rows read and one written per token."""
    d, T, k, N = w.d_model, w.T, w.top_k, w.n_experts
    esz = 2 if w.dtype == "bf16" else 4
    g1, g2, _ = layer_work(w, kept_rows, touched)
    if w.dtype == "f32":
        return {"bound": "latency", "note": "fp32 layer of a few MFLOP: launch-latency bound", "frac": None}
    if stage in ("gemm1", "gemm2"):
        fl = g1 if stage == "gemm1" else g2
        a = fl / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": a, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": a / pk["bf16_tflops"], "flops": fl}
    if stage == "router+aux":
        b = T * d * esz + N * d * 4 + T * k * 8
    elif stage == "dispatch+gather":
        dropped_tok = max(0, T - kept_rows) if k == 1 else 0
        b = T * k * 8 + T * k * 5 + kept_rows * 8 + 2 * kept_rows * d * esz + dropped_tok * d * esz
    else:
        b = T * k * d * esz + T * d * esz
    a = b / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": a, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": a / pk["hbm_gbs"],
            "bytes": b}


# ------------------------------------------------------------ one workload ----

STAGES = ("router+aux", "dispatch+gather", "gemm1", "gemm2", "combine")


def time_layer(layer, x, K, warmup, local, graph=True):
    """W warm-up forwards, then K forwards with stage events (eager) and K
    replays of a CUDA graph of one forward; returns timings and clocks."""
    import numpy as np
    import torch

    from mixture_experts_sparse_b200 import native as nat
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        nat.check(layer.forward(x, routing_outputs=False))
    torch.cuda.synchronize()
    nat.check(nat.moe_read_device_status(layer.ws))
    rev = RawEvents()
    ev = [[rev.create() for _ in range(6)] for _ in range(K)]
    start, stop = rev.create(), rev.create()
    w_ = layer.w
    sampler = ClockSampler(local)
    sampler.start()
    rev.record(start, stream)
    for i in range(K):
        nat.check(nat.moe_forward_events(layer.cfg, x, w_["w_r"], w_["b_r"], w_["w1"], w_["b1"], w_["w3"],
                                         w_["b3"], w_["w2"], w_["b2"], layer.out, offsets=layer.offsets,
                                         kept=layer.kept, aux=layer.aux, ws=layer.ws, events=ev[i]))
    rev.record(stop, stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    nat.check(nat.moe_read_device_status(layer.ws))
    eager_ms = rev.ms(start, stop)
    stage = np.array([[rev.ms(ev[i][j], ev[i][j + 1]) for j in range(5)] for i in range(K)])
    rev.close()
    graph_ms = None
    if graph:
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
        sampler = ClockSampler(local)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sampler.start()
        g0.record(stream)
        for _ in range(K):
            g.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        clocks = sampler.stop()
        nat.check(nat.moe_read_device_status(layer.ws))
        graph_ms = g0.elapsed_time(g1)
        del g
    return dict(eager_ms=eager_ms, graph_ms=graph_ms, stage_ms=stage.mean(axis=0), clocks=clocks)


def workload_summary(w, C, t, kept_rows, touched, pk):
    """Per-workload block: ms/step, tokens/s, layer and dominant-kernel roofline."""
    K = t["K"]
    main_ms = t["graph_ms"] if t["graph_ms"] is not None else t["eager_ms"]
    step_ms = main_ms / K
    g1, g2, bytes_alg = layer_work(w, kept_rows, touched)
    roof_burst = max((g1 + g2) / (pk["bf16_tflops"] * 1e12), bytes_alg / (pk["hbm_gbs"] * 1e9)) * 1e3
    sus = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    roof_sus = max((g1 + g2) / (sus * 1e12), bytes_alg / (pk["hbm_gbs"] * 1e9)) * 1e3
    st = {name: float(v) for name, v in zip(STAGES, t["stage_ms"])}
    if w.dtype == "bf16" and w.top_k == 1:
        st.pop("combine")   # fused into the second GEMM's epilogue
    dom = max(st, key=st.get)
    rl = stage_roofline(dom, w, kept_rows, touched, st[dom], pk)
    rl["kernel"] = dom
    rl["avg_launch_ms"] = st[dom]
    return {
        "T": w.T, "d_model": w.d_model, "d_ff": w.d_ff, "n_experts": w.n_experts, "top_k": w.top_k,
        "capacity_factor": w.capacity_factor, "capacity": C, "act": w.act, "dtype": w.dtype,
        "ms_per_step": step_ms, "tokens_per_s": w.T * K / (main_ms * 1e-3), "steps": K,
        "launch": "CUDA graph replay of moe_forward" if t["graph_ms"] is not None else "moe_forward calls",
        "eager_ms_per_step": t["eager_ms"] / K,
        "kept_assignments": kept_rows, "touched_experts": touched,
        "layer_roofline": {"flops": g1 + g2, "bytes": bytes_alg, "roofline_ms": roof_burst,
                           "frac": roof_burst / step_ms, "frac_vs_sustained_bf16": roof_sus / step_ms,
                           "bound": "tensor" if (g1 + g2) / (pk["bf16_tflops"] * 1e12) >=
                                    bytes_alg / (pk["hbm_gbs"] * 1e9) else "hbm"},
        "dominant_kernel": rl,
        "stages_ms": st,
        "clocks": t["clocks"],
    }


def time_backward(w, L, layer, x, C, K, warmup, pk):
    """The layer's backward on the same batch: the expert FFN backward
    (moe_expert_backward: recompute of the first GEMM, dA, dx, dW1/dW3, dW2 and
    the bias sums) and the router backward (moe_gate_grad + moe_router_backward).
    Algorithmic FLOPs of the expert backward: dA, dx, dW1 (dW3), dW2 =
    (4 ReLU | 6 SwiGLU) x 2 d d_ff per kept row; the recompute is not counted."""
    import torch

    from mixture_experts_sparse_b200 import native as nat
    T, d, dff, N, k = w.T, w.d_model, w.d_ff, w.n_experts, w.top_k
    dev = dict(device="cuda")
    cfg = layer.cfg
    R = max(1, min(k * T, N * C))
    i32, f32 = torch.int32, torch.float32
    idx = torch.empty(T, k, dtype=i32, **dev)
    gate = torch.empty(T, k, dtype=f32, **dev)
    probs = torch.empty(T, N, dtype=f32, **dev)
    pos = torch.empty(T, k, dtype=i32, **dev)
    drop = torch.empty(T, k, dtype=torch.uint8, **dev)
    counts = torch.empty(k, N, dtype=i32, **dev)
    kept = torch.empty(N, dtype=i32, **dev)
    offsets = torch.empty(N + 1, dtype=i32, **dev)
    row_token = torch.empty(R, dtype=i32, **dev)
    row_gate = torch.empty(R, dtype=f32, **dev)
    xe = torch.empty(R, d, dtype=torch.bfloat16, **dev)
    ye = torch.empty(R, d, dtype=torch.bfloat16, **dev)
    fv = torch.empty(N, dtype=torch.float64, **dev)
    Wl = layer.w
    nat.check(nat.moe_route(cfg, x, Wl["w_r"], Wl["b_r"], idx, gate, probs, fv, None, None, layer.ws))
    nat.check(nat.moe_dispatch(cfg, x, idx, gate, pos, drop, counts, kept, offsets, row_token, row_gate, xe,
                               layer.ws))
    nat.check(nat.moe_expert_ffn(cfg, xe, offsets, Wl["w1"], Wl["b1"], Wl["w3"], Wl["b3"], Wl["w2"], Wl["b2"], ye,
                                 layer.ws))
    dout = (0.1 * torch.randn(T, d, **dev)).to(torch.bfloat16)
    nb = nat.moe_expert_backward_workspace_bytes(cfg)
    wsb = torch.empty(nb, dtype=torch.uint8, **dev)
    nat.check(nat.moe_workspace_init(wsb))
    sw = w.act == "swiglu"
    dx = torch.empty(T, d, dtype=f32, **dev)
    dw1 = torch.empty(N, dff, d, dtype=f32, **dev)
    dw3 = torch.empty(N, dff, d, dtype=f32, **dev) if sw else None
    dw2 = torch.empty(N, d, dff, dtype=f32, **dev)
    dgate = torch.empty(T, k, dtype=f32, **dev)
    dh = torch.empty(T, N, dtype=f32, **dev)
    dwr = torch.empty(N, d, dtype=f32, **dev)
    dxr = torch.empty(T, d, dtype=f32, **dev)
    stream = torch.cuda.current_stream()

    def expert():
        nat.check(nat.moe_expert_backward(cfg, xe, offsets, row_token, row_gate, idx, pos, drop, dout, Wl["w1"],
                                          Wl["b1"], Wl["w3"], Wl["b3"], Wl["w2"], dx, dw1, None, dw3, None, dw2,
                                          None, wsb))

    def router():
        nat.check(nat.moe_gate_grad(cfg, dout, ye, idx, pos, drop, offsets, dgate))
        nat.check(nat.moe_router_backward(cfg, x, Wl["w_r"], probs, idx, gate, fv, dgate, dh, dwr, None, dxr,
                                          layer.ws))

    out = {}
    for name, fn in (("expert", expert), ("router", router)):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        out[name] = e0.elapsed_time(e1) / K
    nat.check(nat.moe_read_device_status(wsb))
    nat.check(nat.moe_read_device_status(layer.ws))
    kept_rows = int(offsets[-1].item())
    flops = (6 if sw else 4) * 2 * d * dff * kept_rows
    ach = flops / (out["expert"] * 1e-3) / 1e12
    return {"expert_ms": out["expert"], "router_ms": out["router"], "expert_flops": flops,
            "expert_achieved_tflops": ach, "expert_frac": ach / pk["bf16_tflops"],
            "note": "expert backward: recompute of the first GEMM + dA, dx, dW1 (dW3), dW2 on the tensor cores; "
                    "FLOPs count dA, dx and the weight gradients only; router backward on the tensor cores (bf16 x: "
                    "exact three-way bf16 splits of dh and W_r)"}


def build_layer(w, rank, local, x_seed=None):
    import torch

    from mixture_experts_sparse_b200 import inputs
    from mixture_experts_sparse_b200 import native as nat
    from mixture_experts_sparse_b200.layer import MoeLayer, to_device
    C = nat.moe_capacity(w.T, w.n_experts, w.top_k, w.capacity_factor)
    L = inputs.make_workload(w, x_seed=x_seed)
    layer = MoeLayer(w.T, w.d_model, w.d_ff, w.n_experts, w.top_k, C, w.dtype, w.act, L, alpha=w.alpha)
    x = to_device(L["x"])
    torch.cuda.synchronize()
    return L, layer, x, C


def e2e_single(layer, x, K, warmup):
    """Same metric through the C ABI with host buffers: every step copies its
    input from pinned host memory and its output (and aux loss) back; the
    copies of neighbouring steps overlap the forward on their own streams."""
    import torch

    from mixture_experts_sparse_b200 import native as nat
    stream = torch.cuda.current_stream()
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

    def step(i):
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

    def run(n):
        for i in range(n):
            step(i)
        stream.wait_event(ev_out[(n - 1) & 1])
        if n >= 2:
            stream.wait_event(ev_out[(n - 2) & 1])

    run(max(3, min(warmup, 10)))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    run(K)
    e1.record(stream)
    torch.cuda.synchronize()
    nat.check(nat.moe_read_device_status(layer.ws))
    return e0.elapsed_time(e1), x.numel() * x.element_size(), layer.out.numel() * layer.out.element_size() + 8


def cpu_baselines(L, w, seconds):
    """The oracle on the host cores: single-threaded, and over all host threads."""
    v1, n1, dt1 = oracle_tokens_per_s(L, w, seconds, threads=1)
    nt = host_threads()
    single = {"value": v1, "unit": UNIT, "cores": 1, "kind": "oracle",
              "sample": f"prefix sample: the first {n1} of the batch's {w.T} tokens as one routing group (C from "
                        f"the same cf), full layer forward in the single-threaded C oracle, {dt1:.1f} s"}
    if nt <= 1:
        return single
    vm, nm, dtm = oracle_tokens_per_s(L, w, seconds, threads=nt)
    return {"value": vm, "unit": UNIT, "cores": nt, "kind": "oracle",
            "sample": f"prefix sample: the first {nm} of the batch's {w.T} tokens as one routing group (C from the "
                      f"same cf); routing, aux loss and the serial slot claim once, then the per-token expert work "
                      f"of the oracle over {nt} host threads (os.sched_getaffinity at run time), {dtm:.1f} s",
            "single_core": single}


# ------------------------------------------------------------------ main ----

def run_single(args, local):
    import torch

    torch.cuda.set_device(local)
    pk, pk_src = peaks()
    names = [args.workload] + ([] if args.only else [n for n in ORDER if n != args.workload])
    K, W = args.steps, args.warmup
    blocks, head = {}, None
    for name in names:
        w = WORKLOADS[name]
        if args.tokens and name == args.workload:
            w = w.scaled(T=args.tokens)
        L, layer, x, C = build_layer(w, 0, local)
        t = time_layer(layer, x, K, W, local, graph=not args.no_graph)
        t["K"] = K
        kept_rows = int(layer.offsets[-1].item())
        touched = int((layer.kept > 0).sum().item())
        blocks[name] = workload_summary(w, C, t, kept_rows, touched, pk)
        if w.dtype == "bf16" and not args.no_backward:
            blocks[name]["backward"] = time_backward(w, L, layer, x, C, max(3, min(K, 10)), 2, pk)
        if name == args.workload:
            e2e_ms, h2d, d2h = e2e_single(layer, x, K, W)
            cpu = None if args.no_cpu_baseline else cpu_baselines(L, w, args.cpu_seconds)
            head = dict(w=w, C=C, t=t, kept=kept_rows, touched=touched, e2e=(e2e_ms, h2d, d2h), cpu=cpu)
        del layer, x, L
        torch.cuda.empty_cache()

    w, C, t = head["w"], head["C"], head["t"]
    b = blocks[args.workload]
    g1, g2, bytes_alg = layer_work(w, head["kept"], head["touched"])
    gemm1_ms = b["stages_ms"]["gemm1"]
    achieved_tf = g1 / (gemm1_ms * 1e-3) / 1e12
    traffic = None
    tr = NCU_TRAFFIC.get(args.workload)
    if tr and tr.get("src_sha") == gemm_source_sha():
        traffic = tr["bytes_per_launch"]
    main_ms = t["graph_ms"] if t["graph_ms"] is not None else t["eager_ms"]
    e2e_ms, h2d, d2h = head["e2e"]
    launches_per_step = 6 + (0 if (w.dtype == "bf16" and w.top_k == 1) else 1)
    line = {
        "metric": METRIC, "value": job_tokens_per_s(w.T, 1, K, main_ms), "unit": UNIT, "n_gpus": 1, "steps": K,
        "warmup": W, "ms_per_step": main_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "T": w.T, "d_model": w.d_model, "d_ff": w.d_ff,
                   "n_experts": w.n_experts, "top_k": w.top_k, "capacity_factor": w.capacity_factor,
                   "capacity": C, "act": w.act, "router": "fp32",
                   "l2": "inputs larger than L2: x + expert weights = %.0f MB > 126 MB, no flush"
                         % ((w.T * w.d_model * 2 + w.n_experts * (3 if w.act == 'swiglu' else 2)
                             * w.d_model * w.d_ff * 2) / 1e6),
                   "parallelism": "single GPU", "launch": b["launch"], "eager_ms_per_step": b["eager_ms_per_step"],
                   "kept_assignments": head["kept"], "touched_experts": head["touched"]},
        "roofline": {"bound": "tensor", "kernel": "grouped_gemm stage 1 (x W1^T + act)",
                     "achieved": achieved_tf, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved_tf / pk["bf16_tflops"], "traffic": traffic,
                     "peak_source": f"{pk_src} bf16 burst (MEASURED_PEAKS.json bf16_tflops)",
                     "frac_vs_sustained_bf16": achieved_tf / pk.get("bf16_tflops_sustained", pk["bf16_tflops"]),
                     "flops_per_launch": g1, "avg_launch_ms": gemm1_ms},
        "layer_roofline": b["layer_roofline"],
        "stages_ms": b["stages_ms"],
        "cpu_baseline": head["cpu"],
        "e2e": {"value": job_tokens_per_s(w.T, 1, K, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / K,
                "overlap": "copies of neighbouring steps overlap the forward (two copy streams)"},
        "gpu_launches": launches_per_step * K,
        "clocks": t["clocks"],
        "workloads": blocks,
        "peaks": {"source": pk_src, "bf16_tflops": pk["bf16_tflops"], "hbm_gbs": pk["hbm_gbs"],
                  "bf16_tflops_sustained": pk.get("bf16_tflops_sustained")},
    }
    print(json.dumps(line), flush=True)


def run_multi(args, rank, world, local):
    """N ranks: the shards of one routing group (or independent replicas)."""
    import torch
    import torch.distributed as dist

    from mixture_experts_sparse_b200 import native as nat
    from mixture_experts_sparse_b200.layer import to_device
    from mixture_experts_sparse_b200.shard import Shard, rank_all_gather, sharded_forward

    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    try:
        pk, pk_src = peaks()
        w = WORKLOADS[args.workload]
        if args.tokens:
            w = w.scaled(T=args.tokens)
        K, W = args.steps, args.warmup
        stream = torch.cuda.current_stream()
        if args.replicas:
            # one routing group per GPU: its own batch and weights seed, no exchange
            from mixture_experts_sparse_b200 import inputs
            from mixture_experts_sparse_b200.layer import MoeLayer
            C = nat.moe_capacity(w.T, w.n_experts, w.top_k, w.capacity_factor)
            L = inputs.make_workload(w, x_seed=w.seed + 7919 * (rank + 1))
            layer = MoeLayer(w.T, w.d_model, w.d_ff, w.n_experts, w.top_k, C, w.dtype, w.act, L, alpha=w.alpha)
            x = to_device(L["x"])
            dist.barrier()
            t = time_layer(layer, x, K, W, local, graph=not args.no_graph)
            dist.barrier()
            main_ms = max_over_ranks(t["graph_ms"] if t["graph_ms"] is not None else t["eager_ms"], world)
            kept_rows = int(layer.offsets[-1].item())
            touched = int((layer.kept > 0).sum().item())
            gemm_ms = float(t["stage_ms"][2]) + float(t["stage_ms"][3])
            clocks = t["clocks"]
            mode = "replicas: one routing group of T tokens per GPU, no data-path collective"
            out, xin = layer.out, x

            def fwd(xd, od):
                nat.check(nat.moe_forward(layer.cfg, xd, layer.w["w_r"], layer.w["b_r"], layer.w["w1"],
                                          layer.w["b1"], layer.w["w3"], layer.w["b3"], layer.w["w2"],
                                          layer.w["b2"], od, aux=layer.aux, ws=layer.ws))
        else:
            # shards of one routing group of world x T tokens; C is the group's
            from mixture_experts_sparse_b200 import inputs
            C = nat.moe_capacity(w.T * world, w.n_experts, w.top_k, w.capacity_factor)
            L = inputs.make_workload(w, x_seed=w.seed + 7919 * (rank + 1))
            Wd = {k: to_device(L.get(k)) for k in ("w_r", "b_r", "w1", "b1", "w3", "b3", "w2", "b2")}
            shard = Shard(w.T, w.d_model, w.d_ff, w.n_experts, w.top_k, C, w.dtype, w.act, Wd, alpha=w.alpha)
            x = to_device(L["x"])
            gather = rank_all_gather()
            ev = {}

            def mark(name):
                if name in ev:
                    ev[name].record(stream)

            for _ in range(W):
                sharded_forward([shard], [x], gather, first_index=rank)
            torch.cuda.synchronize()
            nat.check(nat.moe_read_device_status(shard.ws))
            e_ffn = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            sampler = ClockSampler(local)
            dist.barrier()
            torch.cuda.synchronize()
            sampler.start()
            s0.record(stream)
            for i in range(K):
                ev["experts"], ev["experts_done"] = e_ffn[i]
                sharded_forward([shard], [x], gather, first_index=rank, mark=mark)
            s1.record(stream)
            torch.cuda.synchronize()
            dist.barrier()
            clocks = sampler.stop()
            nat.check(nat.moe_read_device_status(shard.ws))
            main_ms = max_over_ranks(s0.elapsed_time(s1), world)
            gemm_ms = sum(a.elapsed_time(b) for a, b in e_ffn) / K
            kept_rows = int(shard.offsets[-1].item())
            touched = int((shard.kept > 0).sum().item())
            mode = (f"one routing group of {world} x {w.T} tokens split over {world} GPUs: per-expert claim counts "
                    f"all-gathered over NCCL (shard.sharded_forward), result identical to one GPU over the group")
            out, xin = shard.out, x

            def fwd(xd, od):
                outs, _, _, _ = sharded_forward([shard], [xd], gather, first_index=rank)
                od.copy_(outs[0])

        # end to end: host input -> device -> forward -> host output, every step
        xh = torch.empty(xin.shape, dtype=xin.dtype).pin_memory()
        xh.copy_(xin.cpu())
        oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        xd, od = torch.empty_like(xin), torch.empty_like(out)
        for _ in range(3):
            xd.copy_(xh, non_blocking=True)
            fwd(xd, od)
            oh.copy_(od, non_blocking=True)
        torch.cuda.synchronize()
        dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            xd.copy_(xh, non_blocking=True)
            fwd(xd, od)
            oh.copy_(od, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)

        g1, g2, _ = layer_work(w, kept_rows, touched)
        ach = (g1 + g2) / (gemm_ms * 1e-3) / 1e12
        if rank == 0:
            line = {
                "metric": METRIC, "value": job_tokens_per_s(w.T, world, K, main_ms), "unit": UNIT, "n_gpus": world,
                "steps": K, "warmup": W, "ms_per_step": main_ms / K, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
                "config": {"workload": w.name, "T_per_gpu": w.T, "d_model": w.d_model, "d_ff": w.d_ff,
                           "n_experts": w.n_experts, "top_k": w.top_k, "capacity_factor": w.capacity_factor,
                           "capacity": C, "act": w.act, "router": "fp32", "parallelism": mode,
                           "l2": "inputs larger than L2, no flush"},
                "roofline": {"bound": "tensor", "kernel": "grouped_gemm stages 1 + 2 (rank 0)", "achieved": ach,
                             "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": ach / pk["bf16_tflops"],
                             "traffic": None, "peak_source": f"{pk_src} bf16 burst"},
                "cpu_baseline": None,
                "e2e": {"value": job_tokens_per_s(w.T, world, K, e2e_ms), "unit": UNIT,
                        "h2d_bytes_per_step": xin.numel() * xin.element_size(),
                        "d2h_bytes_per_step": out.numel() * out.element_size(), "ms_per_step": e2e_ms / K},
                "gpu_launches": (12 if not args.replicas else 7) * K,
                "clocks": clocks,
            }
            print(json.dumps(line), flush=True)
    finally:
        torch.cuda.synchronize()
        dist.destroy_process_group()


def run_reference(args, rank, world):
    if rank != 0:
        return
    from mixture_experts_sparse_b200 import inputs
    from oracle import capacity

    w = WORKLOADS[args.workload]
    if args.tokens:
        w = w.scaled(T=args.tokens)
    L = inputs.make_workload(w)
    C = capacity(w.T, w.n_experts, w.top_k, w.capacity_factor)
    nt = host_threads()
    # size one step so the whole run stays within a few minutes
    per_step = max(0.5, min(6.0, args.reference_budget_s / (args.steps + args.warmup)))
    _, n, _ = oracle_tokens_per_s(L, w, per_step, threads=nt)
    for _ in range(args.warmup):
        oracle_forward_seconds(L, w, n, nt)
    el = sum(oracle_forward_seconds(L, w, n, nt) for _ in range(args.steps))
    v = n * args.steps / el
    line = {
        "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": w.name, "T": w.T, "d_model": w.d_model, "d_ff": w.d_ff, "n_experts": w.n_experts,
                   "top_k": w.top_k, "capacity_factor": w.capacity_factor, "capacity": C, "act": w.act},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": nt, "kind": "oracle",
                         "sample": f"each step: the first {n} tokens of the batch as one routing group; routing, "
                                   f"aux loss and the serial slot claim, then the oracle's per-token expert work over "
                                   f"{nt} host threads"},
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
    ap.add_argument("--only", action="store_true", help="time only --workload (no per-workload block)")
    ap.add_argument("--replicas", action="store_true",
                    help="N > 1: one independent routing group per GPU instead of one group split over the GPUs")
    ap.add_argument("--tokens", type=int, default=None, help="override the workload's T (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward timing of each workload")
    ap.add_argument("--no-graph", action="store_true", help="time direct moe_forward calls instead of graph replay")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
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
    elif world > 1:
        run_multi(args, rank, world, local)
    else:
        run_single(args, local)


if __name__ == "__main__":
    main()
