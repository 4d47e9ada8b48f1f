"""Throughput of one melded-FP8 linear training step (FALQON hot path) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl falqon|reference]

A step is the whole hot path for one synthetic token batch of the workload:
  quantize X -> forward GEMM -> quantize dY -> adapter grads dB, dA -> dX GEMM
  -> caller's plain SGD on B (two tiny torch ops) -> row-wise proxy update.
All five library phases run in libfalqon's kernels through the C ABI.

Timing: W untimed warm-up steps, then K timed steps.  The step is captured
once per input slot in a CUDA graph and replayed; each timed step is bracketed
by CUDA events on the launching stream and separated from the next by an L2
flush (a 512 MB write and a 192 MB read, outside the events).  The timed region is bracketed by
a barrier and torch.cuda.synchronize() on both sides; with N > 1 every rank
runs an independent replica on its own batch ("replicas only", weak scaling)
and the reported time is the max over ranks.

Per-phase CUDA events give each kernel group's duration; the roofline object
reports the slowest phase against the measured peaks in MEASURED_PEAKS.json.
`e2e` repeats the step with the inputs in pinned host memory (H2D copies of X
and dY and D2H copies of Y and dX inside the timed region).  `cpu_baseline`
times the CPU oracle on a bounded sample (rank 0, N = 1).
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from synthetic import WORKLOADS, layer_inputs  # noqa: E402

DEFAULT_WORKLOAD = "llama7b_attn_proj_4096x4096x4096_r64"
METRIC = "melded FP8 linear fwd+bwd+proxy tokens/s; % of FP8 tensor peak / HBM"
FP8_OVER_BF16 = 2.0  # nominal dense FP8 / BF16 tensor throughput ratio on B200


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def max_over_ranks(value: float, device=None) -> float:
    """Max of `value` over all ranks of the default process group (no-op alone)."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"falqon_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------ GPU arm
class Step:
    """Device buffers and the captured step for one workload layer."""

    def __init__(self, wl, layer, torch, F, dev, n_slots=2, seed_offset=0):
        self.torch, self.F, self.dev = torch, F, dev
        self.M, self.N, self.K, self.r = wl.M, layer.N, layer.K, wl.r
        self.lr = wl.lr
        t = torch
        d0 = layer_inputs(wl, layer, step=seed_offset, with_b=True)

        def bf16(bits):
            return t.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(t.bfloat16).to(dev)

        # persistent state of the layer
        self.W = t.from_numpy(d0["W"]).to(dev)
        self.wq = t.empty((self.N, self.K), dtype=t.uint8, device=dev)
        self.s_w = t.empty(1, dtype=t.float32, device=dev)
        self.A = bf16(d0["A"])
        self.B = bf16(d0["B"])
        self.P = t.zeros((self.N, self.K), dtype=t.float32, device=dev)
        self.status = t.zeros(1, dtype=t.int32, device=dev)
        # fresh X / dY per step: a few distinct slots, cycled
        self.X = [bf16(layer_inputs(wl, layer, step=seed_offset + s)["X"]) for s in range(n_slots)]
        self.dY = [bf16(layer_inputs(wl, layer, step=seed_offset + s)["dY"]) for s in range(n_slots)]
        # outputs and intermediates
        self.xq = t.empty((self.M, self.K), dtype=t.uint8, device=dev)
        self.dyq = t.empty((self.M, self.N), dtype=t.uint8, device=dev)
        self.s_x = t.empty(1, dtype=t.float32, device=dev)
        self.s_dy = t.empty(1, dtype=t.float32, device=dev)
        self.amax = t.empty(1, dtype=t.float32, device=dev)
        self.y = t.empty((self.M, self.N), dtype=t.bfloat16, device=dev)
        self.dx = t.empty((self.M, self.K), dtype=t.bfloat16, device=dev)
        self.dA = t.empty((self.r, self.K), dtype=t.bfloat16, device=dev)
        self.dB = t.empty((self.N, self.r), dtype=t.bfloat16, device=dev)
        self.dB_inc = t.empty((self.N, self.r), dtype=t.bfloat16, device=dev)
        self.mask = t.empty(self.N, dtype=t.uint8, device=dev)
        self.n_sel = t.zeros(1, dtype=t.int32, device=dev)

        def ws(op, M, N, K, r):
            n = F.falqon_workspace_size(op, M, N, K, r)
            return t.empty(max(n, 256), dtype=t.uint8, device=dev)

        self.ws_q = ws(F.OP_QUANTIZE, self.M, max(self.N, self.K), 0, 0)
        self.ws_q2 = ws(F.OP_QUANTIZE, self.N, self.K, 0, 0)
        self.ws_bwd = ws(F.OP_LINEAR_BWD, self.M, self.N, self.K, self.r)
        self.ws_p = ws(F.OP_PROXY_UPDATE, 0, self.N, self.K, self.r)
        # initial quantization of the backbone (not part of the step)
        F.falqon_quantize(self.W, codes=self.wq, scale=self.s_w, amax=self.amax,
                          dev_status=self.status, workspace=self.ws_q2)
        # library kernels per step: quantize X (1) + forward (1) + quantize dY (1)
        # + adapter products (T with U, dB with dA: 2) + dX (1) + proxy update and clear (2)
        self.launches_per_step = 1 + 1 + 1 + 2 + 1 + 2

    # one C-ABI call per phase (the caller's SGD: two torch ops)
    PHASES = ("quantX", "fwd", "quantdY", "adapters", "dX", "sgd", "proxy")

    def phase(self, slot, k):
        """Enqueues phase k of one step on the current stream."""
        F, t = self.F, self.torch
        name = self.PHASES[k]
        if name == "quantX":
            F.falqon_quantize(self.X[slot], codes=self.xq, scale=self.s_x, amax=self.amax,
                              dev_status=self.status, workspace=self.ws_q)
        elif name == "fwd":
            F.falqon_linear_fwd(self.xq, self.s_x, self.wq, self.s_w, y=self.y,
                                dev_status=self.status)
        elif name == "quantdY":
            F.falqon_quantize(self.dY[slot], codes=self.dyq, scale=self.s_dy, amax=self.amax,
                              dev_status=self.status, workspace=self.ws_q)
        elif name == "adapters":
            F.falqon_linear_bwd(self.dyq, self.s_dy, self.wq, self.s_w, self.xq, self.s_x, self.A,
                                self.B, dx=None, dA=self.dA, dB=self.dB, dev_status=self.status,
                                workspace=self.ws_bwd)
        elif name == "dX":
            F.falqon_linear_bwd(self.dyq, self.s_dy, self.wq, self.s_w, None, None, None, None,
                                dx=self.dx, dA=None, dB=None, dev_status=self.status)
        elif name == "sgd":
            # the caller's optimizer: plain SGD on B; the proxy receives the increment
            t.mul(self.dB, -self.lr, out=self.dB_inc)
            self.B.add_(self.dB_inc)
        else:
            F.falqon_proxy_update(self.wq, self.s_w, self.P, self.dB_inc, self.A,
                                  row_mask=self.mask, n_selected=self.n_sel,
                                  dev_status=self.status, workspace=self.ws_p)

    def phases(self, slot):
        """Enqueues one whole step."""
        for k in range(len(self.PHASES)):
            self.phase(slot, k)


# FP32 FMA peak of the CUDA cores (the proxy's bound at large r): 148 SMs x 128
# FP32 lanes x 2 flops x 1.965 GHz (the B200's boost clock)
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12

# DRAM traffic per call of a phase: dram__bytes_read.sum + dram__bytes_write.sum
# of every kernel the call launches, from one ncu capture of the bench's own
# workload (the capture command is stored beside the figure).  A figure holds
# only for the kernel sources it was measured on: when a source's hash
# differs, the roofline's traffic is null.
TRAFFIC = {}


def _traffic(phase):
    import hashlib
    t = TRAFFIC.get(phase)
    if not t:
        return None
    for path, digest in t["sources"].items():
        try:
            with open(os.path.join(ROOT, path), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != digest:
                    return None
        except OSError:
            return None
    return t["bytes"]


def _phase_work(st):
    """Algorithmic work and bound of each phase: flops, bytes (each tensor
    once at its storage width), the roofline that bounds it and its kernels."""
    M, N, K, r = st.M, st.N, st.K, st.r
    proxy_flops, proxy_bytes = 2.0 * N * K * r, 9.0 * N * K + 2.0 * r * (N + K)
    # the proxy is bound by the FP32 FMA pipe when its FMA time exceeds its HBM time
    proxy_alu = proxy_flops / (FP32_FMA_TFLOPS * 1e12) > proxy_bytes / (_peaks()["hbm_gbs"] * 1e9)
    return {
        "quantX": {"flops": 0.0, "bytes": 3.0 * M * K, "bound": "hbm",
                   "kernels": "quantize_stream_kernel"},
        "fwd": {"flops": 2.0 * M * N * K, "bytes": M * K + N * K + 2.0 * M * N, "bound": "tensor",
                "kernels": "tc_gemm_kernel (forward)"},
        "quantdY": {"flops": 0.0, "bytes": 3.0 * M * N, "bound": "hbm",
                    "kernels": "quantize_stream_kernel"},
        # each code matrix is read by two products; A, B, dA, dB and the T / U hi-lo pairs
        "adapters": {"flops": 4.0 * M * r * (N + K),
                     "bytes": 2.0 * (M * K + M * N) + 4.0 * r * (N + K) + 16.0 * M * r,
                     "bound": "hbm", "kernels": "skinny_kernel x2 (T^T with U^T, dB^T with dA)"},
        "dX": {"flops": 2.0 * M * N * K, "bytes": M * N + N * K + 2.0 * M * K, "bound": "tensor",
               "kernels": "tc_gemm_kernel (dX)"},
        "sgd": {"flops": 0.0, "bytes": 8.0 * N * r, "bound": None, "kernels": "torch (caller's SGD)"},
        "proxy": {"flops": proxy_flops, "bytes": proxy_bytes, "bound": "alu" if proxy_alu else "hbm",
                  "kernels": "proxy_pipe_kernel + proxy_clear_kernel"},
    }


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import fp8_quantized_lora_b200 as F

    ws, rank, local = _dist()
    if ws > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    F.lib()
    wl = WORKLOADS[args.workload]
    layer = wl.layers[0]
    st = Step(wl, layer, torch, F, dev, n_slots=2, seed_offset=rank * 1000)
    stream = torch.cuda.Stream(device=dev)
    if args.only:
        # one phase alone, eagerly, warm-up + steps times (for profiler captures)
        k = Step.PHASES.index(args.only)
        with torch.cuda.stream(stream):
            st.phases(0)  # one whole step first, so every input of the phase is real data
            for i in range(args.warmup + args.steps):
                st.phase(i % 2, k)
        torch.cuda.synchronize()
        status = int(st.status.item())
        return {"only": args.only, "launches": args.warmup + args.steps, "device_status": status}, rank
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    flush_tail = flush[: 192 << 20].view(torch.int32)

    def l2_flush(i):
        """Evicts L2: a 512 MB write, then a 192 MB read, so that the lines left
        behind are clean and no write-back of the flush lands in the next step."""
        flush.fill_(i & 0xFF)
        flush_tail.sum()

    # capture the step once per input slot
    graphs = []
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for slot in range(2):  # warm the library (attributes, tensor-map encoder) first
            st.phases(slot)
    torch.cuda.synchronize()
    phase_graphs = []  # [slot][phase]: each phase alone, for launch-gap-free attribution
    if not args.no_graph:
        for slot in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                st.phases(slot)
            graphs.append(g)
            per = []
            for k in range(len(Step.PHASES)):
                gk = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gk, stream=stream):
                    st.phase(slot, k)
                per.append(gk)
            phase_graphs.append(per)
    torch.cuda.synchronize()

    def step(i):
        if graphs:
            graphs[i % 2].replay()
        else:
            st.phases(i % 2)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            l2_flush(i)
            step(i)
    torch.cuda.synchronize()
    if int(st.status.item()) != 0:
        raise RuntimeError(f"device status {int(st.status.item())} after warm-up")

    # timed region: per-step events, L2 flush between steps (outside the events)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.25)
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            l2_flush(i)
            starts[i].record()
            step(i)
            ends[i].record()
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    if ws > 1:
        dist.barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(float(np.sum(step_ms)), dev)

    # per-phase timing: each phase replayed from its own graph, back to back,
    # events between the replays; same L2 flush discipline as the timed steps
    names = list(Step.PHASES)
    acc = {n: 0.0 for n in names}
    reps = max(5, min(50, args.steps))
    with torch.cuda.stream(stream):
        for i in range(reps):
            l2_flush(i)
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
            ev[0].record()
            for k in range(len(names)):
                if phase_graphs:
                    phase_graphs[i % 2][k].replay()
                else:
                    st.phase(i % 2, k)
                ev[k + 1].record()
            torch.cuda.synchronize()
            for j, n in enumerate(names):
                acc[n] += ev[j].elapsed_time(ev[j + 1])
    phase_ms = {n: acc[n] / reps for n in names}

    # e2e through the C ABI with host buffers (pinned), copies inside the timed
    # region.  Inputs are copied in on one stream, the step runs on the compute
    # stream, outputs are copied out on a third, with two slots of every
    # buffer: the copies of neighbouring steps overlap the step and each other
    # (the link is full duplex).  Events order each slot's reuse.
    hostX = [x.cpu().pin_memory() for x in st.X]
    hostdY = [x.cpu().pin_memory() for x in st.dY]
    ys = [st.y, torch.empty_like(st.y)]
    dxs = [st.dx, torch.empty_like(st.dx)]
    hostY = [torch.empty(st.y.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    hostdX = [torch.empty(st.dx.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    hostSel = [torch.empty(1, dtype=torch.int32).pin_memory() for _ in range(2)]
    sel = [torch.empty_like(st.n_sel) for _ in range(2)]  # each step's count, kept per slot
    e2e_steps = max(3, min(args.steps, 50))
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_out = [torch.cuda.Event() for _ in range(e2e_steps)]
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e_start.record(s_in)
    stream.wait_event(e_start)
    s_out.wait_event(e_start)
    for i in range(e2e_steps):
        k = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[i - 2])  # step i-2 no longer reads slot k's inputs
            st.X[k].copy_(hostX[k], non_blocking=True)
            st.dY[k].copy_(hostdY[k], non_blocking=True)
            ev_in[i].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_out[i - 2])  # slot k's outputs of step i-2 copied out
            st.y, st.dx = ys[k], dxs[k]
            st.phases(k)
            sel[k].copy_(st.n_sel)
            ev_done[i].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[i])
            hostY[k].copy_(ys[k], non_blocking=True)
            hostdX[k].copy_(dxs[k], non_blocking=True)
            hostSel[k].copy_(sel[k], non_blocking=True)
            ev_out[i].record(s_out)
    s_out.wait_event(ev_done[e2e_steps - 1])
    e_end.record(s_out)
    torch.cuda.synchronize()
    st.y, st.dx = ys[0], dxs[0]
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end), dev)
    status = int(st.status.item())
    n_sel = int(st.n_sel.item())
    topk = _time_topk(st, F, torch, stream, l2_flush, args, dev) if args.topk > 0 else None
    e5 = _time_e5m2(st, F, torch, stream, l2_flush, args, dev) if args.e5m2 else None
    folded = _time_folded(st, F, torch, stream, l2_flush, args, dev) if args.folded else None

    tokens_total = wl.M * args.steps * ws
    value = tokens_total / (total_ms / 1e3)
    e2e_value = wl.M * e2e_steps * ws / (e2e_ms / 1e3)
    h2d = 2 * (st.X[0].numel() * 2 + st.dY[0].numel() * 2) // 2
    d2h = st.y.numel() * 2 + st.dx.numel() * 2 + 4

    peaks = _peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    work = _phase_work(st)
    phases = {}
    for n in names:
        ms = phase_ms[n]
        w = work[n]
        tflops = w["flops"] / (ms * 1e-3) / 1e12 if ms > 0 else 0.0
        gbs = w["bytes"] / (ms * 1e-3) / 1e9 if ms > 0 else 0.0
        ph = {"ms": round(ms, 5), "kernels": w["kernels"], "bound": w["bound"],
              "tflops": round(tflops, 2), "gbs": round(gbs, 1),
              "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
        if w["bound"] == "tensor":
            ph["frac_fp8_peak"] = round(tflops / fp8_peak, 4)
        if w["bound"] == "alu":
            ph["frac_fp32_fma_peak"] = round(tflops / FP32_FMA_TFLOPS, 4)
        phases[n] = ph
    # dominant kernel: the library phase with the largest share of the step
    dom = max((n for n in names if work[n]["bound"]), key=lambda n: phase_ms[n])
    b = work[dom]["bound"]
    if b == "tensor":
        roof = {"kernel": work[dom]["kernels"], "phase": dom, "bound": "tensor",
                "achieved": phases[dom]["tflops"], "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                "frac": phases[dom]["frac_fp8_peak"],
                "peak_source": f"{peaks['source']} bf16 burst x {FP8_OVER_BF16} (nominal FP8/BF16)"}
    elif b == "alu":
        roof = {"kernel": work[dom]["kernels"], "phase": dom, "bound": "alu",
                "achieved": phases[dom]["tflops"], "peak": round(FP32_FMA_TFLOPS, 1), "unit": "TFLOP/s",
                "frac": phases[dom]["frac_fp32_fma_peak"],
                "peak_source": "FP32 FMA: 148 SMs x 128 lanes x 2 flops x 1.965 GHz (nominal units and clock)",
                "hbm_frac": phases[dom]["frac_hbm"]}
    else:
        roof = {"kernel": work[dom]["kernels"], "phase": dom, "bound": "hbm",
                "achieved": phases[dom]["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": phases[dom]["frac_hbm"], "peak_source": f"{peaks['source']} copy bandwidth"}
    roof["traffic"] = _traffic(dom)
    if roof["traffic"] is not None:
        roof["traffic_capture"] = TRAFFIC[dom]["capture"]

    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic",
        "config": {"workload": wl.name, "M": wl.M, "N": layer.N, "K": layer.K, "r": wl.r,
                   "global_batch_tokens": wl.M * ws, "parallelism": f"replicas{ws}",
                   "l2": "flushed between timed steps (512 MB write + 192 MB read, outside the events)",
                   "cuda_graph": not args.no_graph, "lr": wl.lr},
        "roofline": roof,
        "phases": phases,
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": e2e_steps,
                "pipelining": "copy-in, step and copy-out on three streams, two buffer slots"},
        "gpu_launches": st.launches_per_step * args.steps,
        "clocks": clock_info,
        "device_status": status,
        "rows_selected_last_step": n_sel,
        "extra": {"proxy_topk": topk, "e5m2_gradients": e5, "folded_adapters": folded},
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, layer, budget_s=args.cpu_budget)
    if ws > 1:
        dist.destroy_process_group()
    return out, rank


def _graph_phase_times(torch, stream, l2_flush, fns, reps, use_graph=True):
    """Device time (ms) of each enqueueing function in ``fns``: each is
    captured in its own CUDA graph and the graphs are replayed back to back
    with events between them (no host launch gaps inside a phase), L2 flushed
    before every rep outside the events; 3 untimed reps first."""
    with torch.cuda.stream(stream):
        for f in fns:  # warm the library (attributes, tensor-map encoder)
            f()
    torch.cuda.synchronize()
    graphs = []
    if use_graph:
        for f in fns:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                f()
            graphs.append(g)
    torch.cuda.synchronize()
    acc = [0.0] * len(fns)
    with torch.cuda.stream(stream):
        for i in range(3 + reps):
            l2_flush(i)
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
            ev[0].record()
            for k, f in enumerate(fns):
                if graphs:
                    graphs[k].replay()
                else:
                    f()
                ev[k + 1].record()
            torch.cuda.synchronize()
            if i >= 3:
                for k in range(len(fns)):
                    acc[k] += ev[k].elapsed_time(ev[k + 1])
    return [a / reps for a in acc]


def _time_topk(st, F, torch, stream, l2_flush, args, dev):
    """The top-k proxy update over the r rank components (not part of the
    step): a proxy Q [r, N] holding the step's last dB_inc added to a copy of
    the step's Wq, k components merged per call."""
    N, K, r = st.N, st.K, st.r
    k = min(args.topk, r)
    wq = st.wq.clone()
    Q = torch.zeros((r, N), dtype=torch.float32, device=dev)
    mask = torch.empty(r, dtype=torch.uint8, device=dev)
    cnt = torch.zeros(1, dtype=torch.int32, device=dev)
    wsz = F.falqon_workspace_size(F.OP_PROXY_UPDATE_TOPK, 0, N, K, r)
    ws = torch.empty(max(wsz, 256), dtype=torch.uint8, device=dev)
    reps = max(5, min(50, args.steps))

    def call():
        F.falqon_proxy_update_topk(wq, st.s_w, Q, st.dB_inc, st.A, k, comp_mask=mask, n_selected=cnt,
                                   dev_status=st.status, workspace=ws)
    (ms,) = _graph_phase_times(torch, stream, l2_flush, [call], reps, not args.no_graph)
    flops = 2.0 * N * K * k
    nbytes = 2.0 * N * K + 8.0 * r * N + 2.0 * r * N + 2.0 * r * K  # Wq read + write, Q, dB_inc, A
    return {"k": k, "r": r, "ms": round(ms, 5), "components_merged": int(cnt.item()),
            "fp32_fma_tflops": round(flops / (ms * 1e-3) / 1e12, 2),
            "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
            "kernels": "topk_accum_kernel + topk_select_kernel + topk_merge_kernel + topk_clear_kernel",
            "timing": "CUDA graph replay, events on the launching stream",
            "device_status": int(st.status.item())}


def _time_e5m2(st, F, torch, stream, l2_flush, args, dev):
    """The backward with E5M2 gradients (not part of the step): quantize dY
    to E5M2, then the adapter products and dX reading it."""
    dyq = torch.empty_like(st.dyq)
    s_dy = torch.empty(1, dtype=torch.float32, device=dev)
    dA, dB, dx = torch.empty_like(st.dA), torch.empty_like(st.dB), torch.empty_like(st.dx)
    names = ("quantdY", "adapters", "dX")
    reps = max(5, min(50, args.steps))
    fns = [
        lambda: F.falqon_quantize(st.dY[0], codes=dyq, scale=s_dy, amax=st.amax, dev_status=st.status,
                                  workspace=st.ws_q, fmt="e5m2"),
        lambda: F.falqon_linear_bwd(dyq, s_dy, st.wq, st.s_w, st.xq, st.s_x, st.A, st.B, dx=None, dA=dA,
                                    dB=dB, dev_status=st.status, workspace=st.ws_bwd, dy_fmt="e5m2"),
        lambda: F.falqon_linear_bwd(dyq, s_dy, st.wq, st.s_w, None, None, None, None, dx=dx, dA=None,
                                    dB=None, dev_status=st.status, dy_fmt="e5m2"),
    ]
    ms = _graph_phase_times(torch, stream, l2_flush, fns, reps, not args.no_graph)
    out = {n: round(t, 5) for n, t in zip(names, ms)}
    M, N, K = st.M, st.N, st.K
    out["dX_tflops"] = round(2.0 * M * N * K / (out["dX"] * 1e-3) / 1e12, 1)
    out["unit"] = "ms per call"
    out["timing"] = "CUDA graph replay per call, events on the launching stream"
    out["device_status"] = int(st.status.item())
    return out


def _time_folded(st, F, torch, stream, l2_flush, args, dev):
    """Quantized adapters folded into the backbone GEMMs (not part of the
    step): quantize B, the forward with T's columns, then the dX GEMM with
    U's columns and the dB / dA launch; A is frozen and quantized once,
    outside the timing."""
    aq, s_a, _ = F.falqon_quantize(st.A, dev_status=st.status)
    bq = torch.empty((st.N, st.r), dtype=torch.uint8, device=dev)
    s_b = torch.empty(1, dtype=torch.float32, device=dev)
    amax = torch.empty(1, dtype=torch.float32, device=dev)
    ws_b = torch.empty(max(F.falqon_workspace_size(F.OP_QUANTIZE, st.N, st.r), 256), dtype=torch.uint8,
                       device=dev)
    t_saved = torch.empty(F.falqon_workspace_size(F.OP_FOLDED_T, st.M, 0, 0, st.r), dtype=torch.uint8,
                          device=dev)
    ws_u = torch.empty(F.falqon_workspace_size(F.OP_LINEAR_BWD_FOLDED, st.M, st.N, st.K, st.r),
                       dtype=torch.uint8, device=dev)
    y, dx = torch.empty_like(st.y), torch.empty_like(st.dx)
    dA, dB = torch.empty_like(st.dA), torch.empty_like(st.dB)
    names = ("quantB", "fwd_T", "bwd")
    reps = max(5, min(50, args.steps))
    fns = [
        lambda: F.falqon_quantize(st.B, codes=bq, scale=s_b, amax=amax, dev_status=st.status, workspace=ws_b),
        lambda: F.falqon_linear_fwd_folded(st.xq, st.s_x, st.wq, st.s_w, aq, s_a, y=y, t_saved=t_saved,
                                           dev_status=st.status),
        lambda: F.falqon_linear_bwd_folded(st.dyq, st.s_dy, st.wq, st.s_w, bq, s_b, st.xq, st.s_x, t_saved,
                                           st.r, dx=dx, dA=dA, dB=dB, dev_status=st.status, workspace=ws_u),
    ]
    ms = _graph_phase_times(torch, stream, l2_flush, fns, reps, not args.no_graph)
    out = {n: round(t, 5) for n, t in zip(names, ms)}
    out["total"] = round(sum(ms), 5)
    out["unit"] = "ms per call"
    out["timing"] = "CUDA graph replay per call, events on the launching stream"
    out["kernels"] = ("amax_partial_kernel + quantize_cast_kernel (B); tc_gemm_kernel with T columns; "
                      "tc_gemm_kernel (dX) with U columns + skinny_kernel (dB^T with dA)")
    out["device_status"] = int(st.status.item())
    return out


# ------------------------------------------------------------------ CPU oracle
class _OracleData:
    """Inputs of the oracle arm, generated once: two X / dY slots and the backbone."""

    def __init__(self, O, wl, layer):
        self.slots = [layer_inputs(wl, layer, step=s, with_b=True) for s in range(2)]
        self.wq, self.s_w, _, _ = O.quantize(self.slots[0]["W"])


def _oracle_sample_step(O, wl, layer, data, tokens, proxy_rows, step):
    """One oracle step on a bounded sample: `tokens` rows of X and dY through
    quantize / forward / dX / dB / dA, and `proxy_rows` rows of the proxy update."""
    d = data.slots[step % 2]
    X, dY = np.ascontiguousarray(d["X"][:tokens]), np.ascontiguousarray(d["dY"][:tokens])
    wq, s_w = data.wq, data.s_w
    P = np.zeros((proxy_rows, layer.K), dtype=np.float32)
    t0 = time.perf_counter()
    xq, s_x, _, _ = O.quantize(X)
    O.linear_fwd(xq, s_x, wq, s_w)
    dyq, s_dy, _, _ = O.quantize(dY)
    O.linear_dx(dyq, s_dy, wq, s_w)
    t64, _ = O.adapter_t(xq, s_x, d["A"])
    db = O.adapter_db(dyq, s_dy, t64=t64)
    u64, _ = O.adapter_u(dyq, s_dy, d["B"])
    O.adapter_da(xq, s_x, u64=u64)
    t1 = time.perf_counter()
    dB_inc = O.bf16_round(-wl.lr * O.bf16_to_f64(O.bf16_round(db)))
    O.proxy_update(np.ascontiguousarray(wq[:proxy_rows]), s_w, P,
                   np.ascontiguousarray(dB_inc[:proxy_rows]), d["A"])
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1


def cpu_baseline(wl, layer, budget_s=20.0):
    import oracle as O

    cores = os.cpu_count() or 1
    O.set_threads(cores)
    data = _OracleData(O, wl, layer)
    # a small probe sizes the sample to about budget_s seconds of CPU work
    tokens, prows = 64, 256
    tg, tp = _oracle_sample_step(O, wl, layer, data, tokens, prows, 0)
    scale = max(1.0, budget_s / max(tg + tp, 1e-6))
    tokens = int(min(wl.M, tokens * scale))
    prows = int(min(layer.N, prows * scale))
    tg, tp = _oracle_sample_step(O, wl, layer, data, tokens, prows, 1)
    # per-token and per-proxy-row costs, scaled to the full workload step
    full_s = tg * (wl.M / tokens) + tp * (layer.N / prows)
    return {"value": round(wl.M / full_s, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": (f"{tokens} of {wl.M} tokens through quantize/fwd/dX/dB/dA and {prows} of "
                       f"{layer.N} proxy rows (K={layer.K}, r={wl.r}); per-token and per-row "
                       f"times scaled to one full step"),
            "sample_seconds": round(tg + tp, 3)}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return None, rank
    import oracle as O

    wl = WORKLOADS[args.workload]
    layer = wl.layers[0]
    cores = os.cpu_count() or 1
    O.set_threads(cores)
    tokens, prows = 16, 64
    data = _OracleData(O, wl, layer)
    # size the per-step sample so the whole run stays within ~3 minutes
    tg, tp = _oracle_sample_step(O, wl, layer, data, tokens, prows, 0)
    budget = 150.0 / max(1, args.steps + args.warmup)
    scale = max(0.05, min(4.0, budget / max(tg + tp, 1e-6)))
    tokens = max(1, int(tokens * scale))
    prows = max(1, int(prows * scale))
    for i in range(args.warmup):
        _oracle_sample_step(O, wl, layer, data, tokens, prows, i)
    tot_g = tot_p = 0.0
    for i in range(args.steps):
        g, p = _oracle_sample_step(O, wl, layer, data, tokens, prows, args.warmup + i)
        tot_g += g
        tot_p += p
    per_step = tot_g / args.steps * (wl.M / tokens) + tot_p / args.steps * (layer.N / prows)
    value = wl.M / per_step
    sample = (f"{tokens} of {wl.M} tokens and {prows} of {layer.N} proxy rows per step; "
              f"times scaled to one full step")
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_step * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": wl.name, "M": wl.M, "N": layer.N, "K": layer.K, "r": wl.r},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    return out, rank


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="falqon", choices=["falqon", "reference"])
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--folded", type=int, default=1,
                    help="also time the folded quantized-adapter path (1) or skip it (0)")
    ap.add_argument("--e5m2", type=int, default=1,
                    help="also time the backward with E5M2 gradients (1) or skip it (0)")
    ap.add_argument("--topk", type=int, default=16,
                    help="also time the top-k proxy update merging this many of the r components (0: skip)")
    ap.add_argument("--only", default=None, choices=list(Step.PHASES),
                    help="run one phase alone (warm-up + steps calls) and print no bench line; "
                         "for profiler captures")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        out, rank = run_reference(args)
    else:
        out, rank = run_gpu(args)
    if rank == 0 and out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
