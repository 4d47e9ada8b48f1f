"""Throughput of one melded-FP8 linear training step (FALQON hot path) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--rank R]
                    [--impl falqon|reference]

A step is the whole hot path for one synthetic token batch of the workload,
layer by layer: the forward pass (quantize each activation once, then the
forward GEMM of every layer that reads it), then the backward pass in reverse
layer order (quantize dY, adapter gradients dB and dA, dX GEMM, the caller's
plain SGD on B as two tiny torch ops, row-wise proxy update).  Every library
phase runs in libfalqon's kernels through the C ABI.

Timing: W untimed warm-up steps, then K timed steps replayed back to back
from CUDA graphs (one graph per input slot), bracketed by one pair of CUDA
events on the launching stream, with a barrier and torch.cuda.synchronize()
on both sides.  No L2 flush inside the timed region: the input slots cycled
(4 by default) hold more bytes than the 126 MB L2, and each step pays for its
own reads and for the write-back of what it writes, as in a training loop.
With N > 1 every rank runs an independent replica on its own batch
("replicas only", weak scaling) and the reported time is the max over ranks.

Per-phase times (for attribution only) run the phases of one step in step
order after an L2 flush, with timing events recorded between them as event
nodes of one CUDA graph; the roofline object reports the slowest phase
against the measured peaks in MEASURED_PEAKS.json.  `e2e` repeats the step
with the inputs in pinned host memory (H2D copies of every X and dY and a
D2H read of each layer's selected-row count, or with --e2e-outputs 1 also of
every Y and dX, inside the timed region).  `cpu_baseline` times
the CPU oracle on a bounded sample (rank 0, N = 1).
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

from synthetic import WORKLOADS  # noqa: E402

DEFAULT_WORKLOAD = "llama7b_attn_proj_4096x4096x4096_r64"
METRIC = "melded FP8 linear fwd+bwd+proxy tokens/s; % of FP8 tensor peak / HBM"
FP8_OVER_BF16 = 2.0  # nominal dense FP8 / BF16 tensor throughput ratio on B200
L2_BYTES = 126 * 10**6  # B200 L2


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
def _device_normal(torch, dev, seed, shape, std, dtype):
    """Seeded N(0, std^2) draws made on the device (torch's Philox generator),
    rounded to dtype: the bench's inputs.  The parity tests draw theirs from
    synthetic.gen; the bench's sizes (up to tens of GB for the stack) call for
    a device generator."""
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return (torch.randn(shape, generator=g, device=dev, dtype=torch.float32) * std).to(dtype)


def _seed(wl, *parts):
    from synthetic import stream_seed
    return stream_seed(wl.seed, "/".join([wl.name] + [str(p) for p in parts]))


class LayerState:
    """Persistent state of one layer: backbone codes and scale, adapters,
    proxy, gradients and the caller-owned workspaces."""

    def __init__(self, wl, layer, block, r, torch, F, dev, ws_q):
        t = torch
        self.name, self.block, self.group = layer.name, block, layer.x_group
        self.N, self.K, self.r = layer.N, layer.K, r
        W = _device_normal(t, dev, _seed(wl, block, layer.name, "W"), (self.N, self.K), wl.w_std, t.float32)
        self.wq = t.empty((self.N, self.K), dtype=t.uint8, device=dev)
        self.s_w = t.empty(1, dtype=t.float32, device=dev)
        self.status = t.zeros(1, dtype=t.int32, device=dev)
        amax = t.empty(1, dtype=t.float32, device=dev)
        # initial quantization of the backbone (not part of the step)
        F.falqon_quantize(W, codes=self.wq, scale=self.s_w, amax=amax, dev_status=self.status, workspace=ws_q)
        del W
        self.A = _device_normal(t, dev, _seed(wl, block, layer.name, "A", r), (r, self.K), wl.a_std, t.bfloat16)
        self.B = t.zeros((self.N, r), dtype=t.bfloat16, device=dev)
        self.P = t.zeros((self.N, self.K), dtype=t.float32, device=dev)
        self.dA = t.empty((r, self.K), dtype=t.bfloat16, device=dev)
        self.dB = t.empty((self.N, r), dtype=t.bfloat16, device=dev)
        self.dB_inc = t.empty((self.N, r), dtype=t.bfloat16, device=dev)
        self.mask = t.zeros(self.N, dtype=t.uint8, device=dev)  # no selection before the first step
        self.n_sel = t.zeros(1, dtype=t.int32, device=dev)

        def ws(op, M, N, K, rr):
            n = F.falqon_workspace_size(op, M, N, K, rr)
            return t.empty(max(n, 256), dtype=t.uint8, device=dev)

        self.ws_bwd = ws(F.OP_LINEAR_BWD, wl.M, self.N, self.K, r)
        self.ws_p = ws(F.OP_PROXY_UPDATE, 0, self.N, self.K, r)


class Step:
    """Device buffers and the calls of one step of a workload: every layer of
    every block, the activations shared by the layers of an input group
    quantized once."""

    PHASES = ("quantX", "fwd", "quantdY", "adapters", "dX", "sgd", "proxy")
    # library kernels per call of each phase (the caller's SGD is two torch ops)
    LAUNCHES = {"quantX": 1, "fwd": 1, "quantdY": 1, "adapters": 2, "dX": 1, "sgd": 0, "proxy": 2}

    def __init__(self, wl, torch, F, dev, n_slots=4, seed_offset=0, r=None, n_stack=None, tensor_from=256,
                 grouped=True, defer_clear=True, overlap_sgd=True):
        self.torch, self.F, self.dev = torch, F, dev
        self.overlap_sgd = bool(overlap_sgd)
        self.side = torch.cuda.Stream(device=dev) if self.overlap_sgd else None
        self.grouped = grouped
        t = torch
        self.wl = wl
        self.M, self.r, self.lr = wl.M, (wl.r if r is None else r), wl.lr
        self.n_slots = n_slots
        self.n_stack = n_stack or wl.n_stack
        # the proxy's accumulation: the strict float32 chain, or the tensor cores from rank tensor_from up
        self.proxy_tensor = tensor_from > 0 and self.r >= tensor_from
        self.proxy_flags = F.PROXY_ACCUMULATE | F.PROXY_SELECT | (F.PROXY_TENSOR if self.proxy_tensor else 0)
        # the clear of the selected rows carried to the next step through row_mask (not with TENSOR)
        self.defer_clear = bool(defer_clear) and not self.proxy_tensor
        if self.defer_clear:
            self.proxy_flags |= F.PROXY_DEFER_CLEAR
        maxdim = max(max(l.N, l.K) for l in wl.layers)
        # one quantize workspace for every call of the step, initialised once
        self.ws_q = F.workspace(F.OP_QUANTIZE, self.M, maxdim, device=dev)
        self.layers = [LayerState(wl, l, b, self.r, t, F, dev, self.ws_q)
                       for b in range(self.n_stack) for l in wl.layers]
        # input groups (block, x_group) in order of first use, with their K
        self.groups = {}
        for L in self.layers:
            self.groups.setdefault((L.block, L.group), L.K)
        so = seed_offset
        self.X = [{g: _device_normal(t, dev, _seed(wl, g[0], g[1], "X", so + s), (self.M, K), wl.x_std, t.bfloat16)
                   for g, K in self.groups.items()} for s in range(n_slots)]
        self.dY = [[_device_normal(t, dev, _seed(wl, L.block, L.name, "dY", so + s), (self.M, L.N), wl.dy_std,
                                   t.bfloat16) for L in self.layers] for s in range(n_slots)]
        # codes and scales of every activation (kept from the forward for the backward)
        self.xq = {g: t.empty((self.M, K), dtype=t.uint8, device=dev) for g, K in self.groups.items()}
        self.s_x = {g: t.empty(1, dtype=t.float32, device=dev) for g in self.groups}
        # per-shape outputs, reused across layers: nothing downstream reads them
        self.y = {n: t.empty((self.M, n), dtype=t.bfloat16, device=dev) for n in {L.N for L in self.layers}}
        self.dx = {k: t.empty((self.M, k), dtype=t.bfloat16, device=dev) for k in {L.K for L in self.layers}}
        self.dyq = {n: t.empty((self.M, n), dtype=t.uint8, device=dev) for n in {L.N for L in self.layers}}
        self.s_dy = t.empty(1, dtype=t.float32, device=dev)
        self.amax = t.empty(1, dtype=t.float32, device=dev)
        self.status = t.zeros(1, dtype=t.int32, device=dev)
        self.calls_per_step = {p: 0 for p in self.PHASES}
        for _, p, _ in self.calls(0):
            self.calls_per_step[p] += 1
        self.launches_per_step = sum(self.LAUNCHES[p] * n for p, n in self.calls_per_step.items())

    @property
    def tokens(self):
        return self.M

    def status_words(self):
        return [self.status] + [L.status for L in self.layers]

    def device_status(self) -> int:
        v = 0
        for s in self.status_words():
            v |= int(s.item())
        return v

    def calls(self, slot, outs=None):
        """The step as (layer, phase, enqueue function) in execution order.
        outs: optional (ys, dxs), per-layer output tensors in place of the
        shared per-shape ones."""
        F, t = self.F, self.torch
        X, dY = self.X[slot], self.dY[slot]
        yo = (lambda j, L: outs[0][j]) if outs else (lambda j, L: self.y[L.N])
        xo = (lambda j, L: outs[1][j]) if outs else (lambda j, L: self.dx[L.K])
        out = []
        seen = set()
        for jf, L in enumerate(self.layers):  # forward pass
            g = (L.block, L.group)
            if g in seen:
                continue
            seen.add(g)
            out.append((L, "quantX", lambda g=g: F.falqon_quantize(
                X[g], codes=self.xq[g], scale=self.s_x[g], amax=self.amax, dev_status=self.status,
                workspace=self.ws_q)))
            # every layer of the group reads the same codes: one grouped launch (up to three)
            members = [(j, M_) for j, M_ in enumerate(self.layers) if (M_.block, M_.group) == g]
            for c0 in range(0, len(members), 3 if self.grouped else 1):
                part = members[c0:c0 + (3 if self.grouped else 1)]
                if len(part) == 1:
                    j, M_ = part[0]
                    out.append((M_, "fwd", lambda M_=M_, g=g, y=yo(j, M_): F.falqon_linear_fwd(
                        self.xq[g], self.s_x[g], M_.wq, M_.s_w, y=y, dev_status=M_.status)))
                else:
                    out.append((part[0][1], "fwd", lambda part=part, g=g, ys=[yo(j, M_) for j, M_ in part]:
                                F.falqon_linear_fwd_grouped(self.xq[g], self.s_x[g], [M_.wq for _, M_ in part],
                                                            [M_.s_w for _, M_ in part], ys=ys,
                                                            dev_status=part[0][1].status)))
        for j in range(len(self.layers) - 1, -1, -1):  # backward pass, last layer first
            L = self.layers[j]
            g = (L.block, L.group)
            dyq = self.dyq[L.N]
            out.append((L, "quantdY", lambda j=j, L=L, dyq=dyq: F.falqon_quantize(
                dY[j], codes=dyq, scale=self.s_dy, amax=self.amax, dev_status=self.status, workspace=self.ws_q)))
            out.append((L, "adapters", lambda L=L, g=g, dyq=dyq: F.falqon_linear_bwd(
                dyq, self.s_dy, L.wq, L.s_w, self.xq[g], self.s_x[g], L.A, L.B, dx=None, dA=L.dA, dB=L.dB,
                dev_status=L.status, workspace=L.ws_bwd)))
            out.append((L, "dX", lambda L=L, dyq=dyq, dx=xo(j, L): F.falqon_linear_bwd(
                dyq, self.s_dy, L.wq, L.s_w, None, None, None, None, dx=dx, dA=None, dB=None,
                dev_status=L.status)))

            def sgd(L=L):  # the caller's optimizer: plain SGD on B; the proxy receives the increment
                t.mul(L.dB, -self.lr, out=L.dB_inc)
                L.B.add_(L.dB_inc)
            out.append((L, "sgd", sgd))
            out.append((L, "proxy", lambda L=L: F.falqon_proxy_update(
                L.wq, L.s_w, L.P, L.dB_inc, L.A, flags=self.proxy_flags, row_mask=L.mask, n_selected=L.n_sel,
                dev_status=L.status, workspace=L.ws_p)))
        return out

    def run(self, slot, phase=None, outs=None):
        """Enqueues the whole step (or only the calls of one phase) on the current stream.
        In a whole step the caller's SGD on B, which dX does not read, runs on a
        second stream beside dX (forked after the adapter products, joined
        before the proxy update that reads its increment) when overlap_sgd is set."""
        t = self.torch
        main = t.cuda.current_stream()
        pending = None
        for _, p, f in self.calls(slot, outs):
            if phase is not None and p != phase:
                continue
            if phase is None and p == "sgd" and self.overlap_sgd:
                fork = t.cuda.Event()
                fork.record(main)
                self.side.wait_event(fork)
                with t.cuda.stream(self.side):
                    f()
                pending = t.cuda.Event()
                pending.record(self.side)
                continue
            if p == "proxy" and pending is not None:
                main.wait_event(pending)
                pending = None
            f()
        if pending is not None:
            main.wait_event(pending)


# FP32 FMA peak of the CUDA cores (the proxy's bound at large r): 148 SMs x 128
# FP32 lanes x 2 flops x 1.965 GHz (the B200's boost clock)
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12

# DRAM traffic per call of a phase: dram__bytes_read.sum + dram__bytes_write.sum
# of every kernel the call launches, from one ncu capture of the bench's own
# workload (the capture command is stored beside the figure).  A figure holds
# only for the kernel sources it was measured on: when a source's hash
# differs, the roofline's traffic is null.
TRAFFIC = {
    "proxy": {
        "workload": "llama7b_attn_proj_4096x4096x4096_r64", "r": 64, "defer_clear": True,
        "bytes": 17914624 + 13597440,
        "kernels": ("proxy_ws_kernel<1> (proxy_clear_kernel, which writes the row mask and the "
                    "count, not captured)"),
        "capture": ("ncu --set full --clock-control none -k regex:proxy_ws -s 2 -c 1 python bench.py "
                    "--only proxy --steps 3 --warmup 3 --no-cpu-baseline: dram__bytes_read.sum "
                    "17.91 MB + dram__bytes_write.sum 13.60 MB; with the deferred clear the rows the "
                    "previous call selected are not read, and most of P' is still in L2 when the "
                    "launch ends"),
        "sources": {
            "fp8_quantized_lora_b200/csrc/proxy.cu":
                "bed6522e23166124fb41f662a8d32b2ea570cb2fe8aa84c89171d835e80f3c98",
            "fp8_quantized_lora_b200/csrc/ptx.cuh":
                "ff1913ffafac4e65526e4c62e66cb1811fd632c060b2a9c5595e488983d60665",
            "fp8_quantized_lora_b200/csrc/codes.cuh":
                "0daacdb7c252d2163d86f9b6ef6c40a2522e5c60497bc5d5b377385ce0f5b1b0",
        },
    },
}


def _traffic(phase, st):
    """The captured DRAM bytes of one call of ``phase``, or None when the
    capture was of another workload, rank or clear mode, or of other kernel
    sources."""
    import hashlib
    t = TRAFFIC.get(phase)
    if not t or t["workload"] != st.wl.name or t["r"] != st.r or t["defer_clear"] != st.defer_clear:
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
    """Algorithmic work and bound of each phase of one layer (st: M, N, K, r):
    flops, bytes (each tensor once at its storage width), the roofline that
    bounds it and its kernels."""
    M, N, K, r = st.M, st.N, st.K, st.r
    proxy_flops, proxy_bytes = 2.0 * N * K * r, 9.0 * N * K + 2.0 * r * (N + K)
    # the proxy is bound by the FP32 FMA pipe when its FMA time exceeds its HBM time
    proxy_alu = proxy_flops / (FP32_FMA_TFLOPS * 1e12) > proxy_bytes / (_peaks()["hbm_gbs"] * 1e9)
    return {
        "quantX": {"flops": 0.0, "bytes": 3.0 * M * K, "bound": "hbm",
                   "kernels": "quantize_stream_kernel"},
        "fwd": {"flops": 2.0 * M * N * K, "bytes": M * K + N * K + 2.0 * M * N, "bound": "tensor",
                "kernels": "tc_gemm_pair_kernel (forward)"},
        "quantdY": {"flops": 0.0, "bytes": 3.0 * M * N, "bound": "hbm",
                    "kernels": "quantize_stream_kernel"},
        # each code matrix is read by two products; A, B, dA, dB and the T / U hi-lo pairs
        "adapters": {"flops": 4.0 * M * r * (N + K),
                     "bytes": 2.0 * (M * K + M * N) + 4.0 * r * (N + K) + 16.0 * M * r,
                     "bound": "hbm", "kernels": "skinny_kernel x2 (T^T with U^T, dB^T with dA)"},
        "dX": {"flops": 2.0 * M * N * K, "bytes": M * N + N * K + 2.0 * M * K, "bound": "tensor",
               "kernels": "tc_gemm_pair_kernel (dX)"},
        "sgd": {"flops": 0.0, "bytes": 8.0 * N * r, "bound": None, "kernels": "torch (caller's SGD)"},
        "proxy": {"flops": proxy_flops, "bytes": proxy_bytes, "bound": "alu" if proxy_alu else "hbm",
                  "kernels": "proxy_ws_kernel + proxy_clear_kernel"},
    }


def _step_work(st):
    """_phase_work summed over one step: every layer's products, every
    activation group's quantization once (its layers share the codes); calls
    as the step issues them (a grouped forward is one call)."""
    import types

    tot = {}

    def add(p, w):
        e = tot.setdefault(p, {"flops": 0.0, "bytes": 0.0, "bound": w["bound"], "kernels": w["kernels"],
                               "calls": st.calls_per_step[p]})
        e["flops"] += w["flops"]
        e["bytes"] += w["bytes"]
    for L in st.layers:
        w = _phase_work(types.SimpleNamespace(M=st.M, N=L.N, K=L.K, r=st.r))
        for p in Step.PHASES:
            if p != "quantX":
                add(p, w[p])
    for K in st.groups.values():
        add("quantX", _phase_work(types.SimpleNamespace(M=st.M, N=K, K=K, r=st.r))["quantX"])
    return tot


def _flusher(torch, dev):
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    flush_tail = flush[: 192 << 20].view(torch.int32)

    def l2_flush(i):
        """Evicts L2: a 512 MB write, then a 192 MB read, so that the lines left
        behind are clean and no write-back of the flush lands in what follows."""
        flush.fill_(i & 0xFF)
        flush_tail.sum()
    return l2_flush


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
    r = args.rank if args.rank else wl.r
    n_stack = args.blocks or wl.n_stack
    # bytes of one slot: every activation group's X and every layer's dY (bf16)
    slot_bytes = n_stack * wl.M * 2 * (sum(k for _, k in {(l.x_group, l.K) for l in wl.layers}) +
                                       sum(l.N for l in wl.layers))
    slots = args.slots or min(8, max(2, -(-(2 * L2_BYTES) // slot_bytes)))
    st = Step(wl, torch, F, dev, n_slots=slots, seed_offset=rank * 1000, r=r, n_stack=n_stack,
              tensor_from=args.proxy_tensor_from, grouped=bool(args.grouped), defer_clear=bool(args.proxy_defer),
              overlap_sgd=bool(args.overlap_sgd))
    stream = torch.cuda.Stream(device=dev)
    if args.only:
        # one phase alone, eagerly, warm-up + steps times (for profiler captures)
        with torch.cuda.stream(stream):
            st.run(0)  # one whole step first, so every input of the phase is real data
            for i in range(args.warmup + args.steps):
                st.run(i % st.n_slots, args.only)
        torch.cuda.synchronize()
        return {"only": args.only, "calls": (args.warmup + args.steps) * st.calls_per_step[args.only],
                "device_status": st.device_status()}, rank
    l2_flush = _flusher(torch, dev)

    # capture the step once per input slot
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for slot in range(min(2, st.n_slots)):  # warm the library (attributes, tensor-map encoder) first
            st.run(slot)
    torch.cuda.synchronize()
    graphs, phase_graphs = [], []  # phase_graphs[slot][phase]: that phase of every layer
    if not args.no_graph:
        for slot in range(st.n_slots):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                st.run(slot)
            graphs.append(g)
        for slot in range(min(2, st.n_slots)):
            phase_graphs.append(_evented_graph(
                torch, stream, [lambda slot=slot, p=p: st.run(slot, p) for p in Step.PHASES]))
    torch.cuda.synchronize()

    def step(i):
        if graphs:
            graphs[i % st.n_slots].replay()
        else:
            st.run(i % st.n_slots)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    torch.cuda.synchronize()
    if st.device_status() != 0:
        raise RuntimeError(f"device status {st.device_status()} after warm-up")

    # timed region: K steps back to back, one event pair (plus one event per step)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    clocks = ClockSampler(local)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.25)
    with torch.cuda.stream(stream):
        evs[0].record()
        for i in range(args.steps):
            step(args.warmup + i)
            evs[i + 1].record()
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    if ws > 1:
        dist.barrier()
    total_ms = max_over_ranks(evs[0].elapsed_time(evs[-1]), dev)
    per_step = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]

    # per-phase attribution: the phases of one step (each of every layer) in
    # step order, one after another, L2 flushed before each rep; timing events
    # between the phases (event nodes inside one graph: no launch gap inside
    # a bracket, and no overlap between phases)
    names = list(Step.PHASES)
    acc = {n: 0.0 for n in names}
    reps = max(5, min(50, args.steps))
    with torch.cuda.stream(stream):
        for i in range(reps):
            l2_flush(i)
            if phase_graphs:
                g, ev = phase_graphs[i % len(phase_graphs)]
                g.replay()
            else:
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
                ev[0].record()
                for k, n in enumerate(names):
                    st.run(i % st.n_slots, n)
                    ev[k + 1].record()
            torch.cuda.synchronize()
            for j, n in enumerate(names):
                acc[n] += ev[j].elapsed_time(ev[j + 1])
    phase_ms = {n: acc[n] / reps for n in names}

    e2e = _time_e2e(st, torch, stream, ws, dev, args) if args.e2e else {"skipped": "--e2e 0"}
    status = st.device_status()
    n_sel = sum(int(L.n_sel.item()) for L in st.layers)
    single = len(st.layers) == 1
    v = _single_view(st) if single else None
    topk = _time_topk(v, F, torch, stream, l2_flush, args, dev) if (args.topk > 0 and single) else None
    e5 = _time_e5m2(v, F, torch, stream, l2_flush, args, dev) if (args.e5m2 and single) else None
    folded = _time_folded(v, F, torch, stream, l2_flush, args, dev) if (args.folded and single) else None
    separate = _time_separate(v, F, torch, stream, l2_flush, args, dev) if (args.separate and single) else None

    tokens_total = st.tokens * args.steps * ws
    value = tokens_total / (total_ms / 1e3)

    peaks = _peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    work = _step_work(st)
    phases = {}
    for n in names:
        ms = phase_ms[n]
        w = work[n]
        tflops = w["flops"] / (ms * 1e-3) / 1e12 if ms > 0 else 0.0
        gbs = w["bytes"] / (ms * 1e-3) / 1e9 if ms > 0 else 0.0
        ph = {"ms": round(ms, 5), "calls": w["calls"], "kernels": w["kernels"], "bound": w["bound"],
              "tflops": round(tflops, 2), "gbs": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
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
    roof["timing"] = ("phases of one step in order after an L2 flush, timing events between them as "
                      "event nodes of one CUDA graph on the launching stream")
    roof["traffic"] = _traffic(dom, st) if single else None
    if roof["traffic"] is not None:
        roof["traffic_kernels"] = TRAFFIC[dom]["kernels"]
        roof["traffic_capture"] = TRAFFIC[dom]["capture"]

    layer0 = st.layers[0]
    slot_bytes = sum(x.numel() * 2 for x in st.X[0].values()) + sum(d.numel() * 2 for d in st.dY[0])
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic",
        "config": {"workload": wl.name, "M": st.M, "r": st.r, "layers": len(st.layers),
                   "blocks": st.n_stack, "shapes": sorted({f"{L.K}->{L.N}" for L in st.layers}),
                   "N": layer0.N, "K": layer0.K,
                   "global_batch_tokens": st.M * ws, "parallelism": f"replicas{ws}",
                   "l2": (f"back to back: no flush; {st.n_slots} input slots cycled "
                          f"({st.n_slots * slot_bytes / 2**20:.0f} MiB of X and dY, above the 126 MB L2)"),
                   "cuda_graph": not args.no_graph, "lr": wl.lr,
                   "proxy_accumulation": ("tensor cores (bf16 products, float32 sums)" if st.proxy_tensor
                                          else "strict float32 FMA chain"),
                   "proxy_clear": ("deferred: row_mask carries it to the next step" if st.defer_clear
                                   else "written every step"),
                   "sgd": "second stream beside dX" if st.overlap_sgd else "in line",
                   "grouped_forward": st.grouped},
        "step_ms_median": round(float(np.median(per_step)), 5),
        "roofline": roof,
        "phases": phases,
        "e2e": e2e,
        "gpu_launches": st.launches_per_step * args.steps,
        "clocks": clock_info,
        "device_status": status,
        "rows_selected_last_step": n_sel,
        "extra": {"proxy_topk": topk, "e5m2_gradients": e5, "folded_adapters": folded,
                  "separate_lora": separate},
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_budget, r=st.r, n_stack=st.n_stack)
    if ws > 1:
        dist.destroy_process_group()
    return out, rank


def _single_view(st):
    """The one layer of a single-layer step, with the step's buffers, for the
    extra rows (top-k, E5M2, folded adapters)."""
    import types

    L = st.layers[0]
    g = (L.block, L.group)
    return types.SimpleNamespace(
        M=st.M, N=L.N, K=L.K, r=st.r, wq=L.wq, s_w=L.s_w, P=L.P, A=L.A, B=L.B, dA=L.dA, dB=L.dB,
        dB_inc=L.dB_inc, xq=st.xq[g], s_x=st.s_x[g], dyq=st.dyq[L.N], s_dy=st.s_dy, dY0=st.dY[0][0], X0=st.X[0][g],
        y=st.y[L.N], dx=st.dx[L.K], ws_bwd=L.ws_bwd, ws_q=st.ws_q, amax=st.amax, status=L.status)


def _time_e2e(st, torch, stream, ws, dev, args):
    """The step through the C ABI with host buffers: every X and dY copied in
    from pinned host memory, and the step's result read back, inside the
    timed region.  The result is the step's metric, each layer's selected-row
    count; with --e2e-outputs 1 every layer's Y and dX are copied out as
    well.  Copy-in, step and copy-out run on three streams with two buffer
    slots, so the copies of neighbouring steps overlap the step and each
    other (the link is full duplex); events order each slot's reuse.  The
    step's calls write every layer's Y and dX into per-slot device buffers."""
    with_outputs = bool(getattr(args, "e2e_outputs", 0))
    in_bytes = sum(x.numel() * 2 for x in st.X[0].values()) + sum(d.numel() * 2 for d in st.dY[0])
    if in_bytes > (4 << 30):
        return {"skipped": f"{in_bytes / 2**30:.1f} GiB of inputs per step: pinned host slots not allocated"}
    nslot = min(2, st.n_slots)
    hostX = [{g: x.cpu().pin_memory() for g, x in st.X[k].items()} for k in range(nslot)]
    hostdY = [[d.cpu().pin_memory() for d in st.dY[k]] for k in range(nslot)]
    # per-step outputs: each layer's Y and dX in their own device and host slots
    ys = [[torch.empty((st.M, L.N), dtype=torch.bfloat16, device=dev) for L in st.layers] for _ in range(nslot)]
    dxs = [[torch.empty((st.M, L.K), dtype=torch.bfloat16, device=dev) for L in st.layers] for _ in range(nslot)]
    hostY = [[torch.empty((st.M, L.N), dtype=torch.bfloat16).pin_memory() for L in st.layers] if with_outputs
             else [] for _ in range(nslot)]
    hostdX = [[torch.empty((st.M, L.K), dtype=torch.bfloat16).pin_memory() for L in st.layers] if with_outputs
              else [] for _ in range(nslot)]
    sel = [torch.empty(len(st.layers), dtype=torch.int32, device=dev) for _ in range(nslot)]
    hostSel = [torch.empty(len(st.layers), dtype=torch.int32).pin_memory() for _ in range(nslot)]
    steps = max(3, min(args.steps, 50))
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(steps)]
    ev_done = [torch.cuda.Event() for _ in range(steps)]
    ev_out = [torch.cuda.Event() for _ in range(steps)]
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    index = {id(L): j for j, L in enumerate(st.layers)}
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    e_start.record(s_in)
    stream.wait_event(e_start)
    s_out.wait_event(e_start)
    for i in range(steps):
        k = i % nslot
        with torch.cuda.stream(s_in):
            if i >= nslot:
                s_in.wait_event(ev_done[i - nslot])  # step i-2 no longer reads slot k's inputs
            for g, x in st.X[k].items():
                x.copy_(hostX[k][g], non_blocking=True)
            for j, d in enumerate(st.dY[k]):
                d.copy_(hostdY[k][j], non_blocking=True)
            ev_in[i].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(ev_in[i])
            if i >= nslot:
                stream.wait_event(ev_out[i - nslot])  # slot k's outputs of step i-2 copied out
            for L, p, f in st.calls(k, (ys[k], dxs[k])):
                f()
                if p == "proxy":
                    j = index[id(L)]
                    sel[k][j:j + 1].copy_(L.n_sel)
            ev_done[i].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[i])
            if with_outputs:
                for j in range(len(st.layers)):
                    hostY[k][j].copy_(ys[k][j], non_blocking=True)
                    hostdX[k][j].copy_(dxs[k][j], non_blocking=True)
            hostSel[k].copy_(sel[k], non_blocking=True)
            ev_out[i].record(s_out)
    s_out.wait_event(ev_done[steps - 1])
    e_end.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end), dev)
    h2d = in_bytes
    d2h = (sum(L.N * st.M * 2 + L.K * st.M * 2 for L in st.layers) if with_outputs else 0) + 4 * len(st.layers)
    return {"value": round(st.M * steps * ws / (e2e_ms / 1e3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "result_read": ("each layer's Y and dX and its selected-row count" if with_outputs
                            else "each layer's selected-row count (the step's metric); Y and dX stay on the device"),
            "pipelining": "copy-in, step and copy-out on three streams, two buffer slots"}


def _evented_graph(torch, stream, fns):
    """One CUDA graph of the enqueueing functions ``fns`` in order, with a
    timing event recorded before the first and after each of them as event
    nodes of the graph: a replay brackets every call on the device with no
    graph-launch gap inside a bracket.  Returns (graph, events)."""
    evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(fns) + 1)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        evs[0].record()
        for k, f in enumerate(fns):
            f()
            evs[k + 1].record()
    return g, evs


def _graph_phase_times(torch, stream, l2_flush, fns, reps, use_graph=True):
    """Device time (ms) of each enqueueing function in ``fns``: all are
    captured in one CUDA graph with timing events between them
    (_evented_graph), and the graph is replayed after an L2 flush (outside
    the events) per rep; 3 untimed reps first."""
    with torch.cuda.stream(stream):
        for f in fns:  # warm the library (attributes, tensor-map encoder)
            f()
    torch.cuda.synchronize()
    graph = _evented_graph(torch, stream, fns) if use_graph else None
    torch.cuda.synchronize()
    acc = [0.0] * len(fns)
    with torch.cuda.stream(stream):
        for i in range(3 + reps):
            l2_flush(i)
            if graph:
                g, ev = graph
                g.replay()
            else:
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
                ev[0].record()
                for k, f in enumerate(fns):
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
            "timing": "one CUDA graph per rep after an L2 flush, timing events as graph nodes",
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
        lambda: F.falqon_quantize(st.dY0, codes=dyq, scale=s_dy, amax=st.amax, dev_status=st.status,
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
    out["timing"] = "one CUDA graph per rep after an L2 flush, timing events as graph nodes between the calls"
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
    ws_b = F.workspace(F.OP_QUANTIZE, st.N, st.r, device=dev)
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
    out["timing"] = "one CUDA graph per rep after an L2 flush, timing events as graph nodes between the calls"
    out["kernels"] = ("amax_partial_kernel + quantize_cast_kernel (B); tc_gemm_kernel with T columns; "
                      "tc_gemm_kernel (dX) with U columns + skinny_kernel (dB^T with dA)")
    out["device_status"] = int(st.status.item())
    return out


def _time_separate(st, F, torch, stream, l2_flush, args, dev):
    """The comparison the pages measure (not part of the step): LoRA kept as
    a separate path beside the same FP8 backbone, in bf16 and with every
    adapter operand quantized to E4M3 (forward and backward of one layer,
    the backbone products included).  The melded step's forward, adapter
    gradients and dX phases are the corresponding FALQON work."""
    M, N, K, r = st.M, st.N, st.K, st.r
    X = st.X0
    out = {"unit": "ms per call", "timing": "one CUDA graph per rep after an L2 flush, timing events as graph nodes between the calls"}
    reps = max(5, min(50, args.steps))
    for name, prec in (("bf16", F.SEPARATE_BF16), ("fp8", F.SEPARATE_FP8)):
        sop = F.OP_SEPARATE_SAVED_FP8 if prec == F.SEPARATE_FP8 else F.OP_SEPARATE_SAVED_BF16
        bop = F.OP_SEPARATE_BWD_FP8 if prec == F.SEPARATE_FP8 else F.OP_SEPARATE_BWD_BF16
        saved = F.workspace(sop, M, N, K, r, device=dev)
        wf = F.workspace(F.OP_SEPARATE_FWD_FP8, M, N, K, r, device=dev) if prec == F.SEPARATE_FP8 else None
        wb = F.workspace(bop, M, N, K, r, device=dev)
        y, dx = torch.empty_like(st.y), torch.empty_like(st.dx)
        dA, dB = torch.empty_like(st.dA), torch.empty_like(st.dB)
        fns = [
            lambda: F.falqon_lora_separate_fwd(prec, st.xq, st.s_x, X, st.wq, st.s_w, st.A, st.B, y=y, saved=saved,
                                               dev_status=st.status, workspace=wf),
            lambda: F.falqon_lora_separate_bwd(prec, st.dyq, st.s_dy, st.dY0, st.wq, st.s_w, st.xq, st.s_x, X, st.A,
                                               st.B, saved, dx=dx, dA=dA, dB=dB, dev_status=st.status, workspace=wb),
        ]
        ms = _graph_phase_times(torch, stream, l2_flush, fns, reps, not args.no_graph)
        out[name] = {"fwd": round(ms[0], 5), "bwd": round(ms[1], 5), "total": round(sum(ms), 5)}
    out["device_status"] = int(st.status.item())
    return out


# ------------------------------------------------------------------ CPU oracle
class _OracleData:
    """Inputs of the oracle arm for one layer shape (K -> N), drawn once with
    synthetic.gen: the backbone (full size, so its scale is the layer's), the
    adapters, and X / dY rows drawn per step at the sample's size."""

    def __init__(self, O, wl, layer, r):
        from synthetic import gen, stream_seed

        self.wl, self.layer, self.r = wl, layer, r
        tag = f"{wl.name}/oracle/{layer.name}"
        W = gen.normal_f32(stream_seed(wl.seed, tag + "/W"), (layer.N, layer.K), wl.w_std)
        self.wq, self.s_w, _, _ = O.quantize(W)
        self.A = gen.normal_bf16_bits(stream_seed(wl.seed, tag + f"/A/r{r}"), (r, layer.K), wl.a_std)
        self.B = gen.normal_bf16_bits(stream_seed(wl.seed, tag + f"/B/r{r}"), (layer.N, r), 1e-3)
        self._tag = tag

    def rows(self, step, tokens):
        from synthetic import gen, stream_seed

        wl, layer = self.wl, self.layer
        X = gen.normal_bf16_bits(stream_seed(wl.seed, self._tag + f"/X/{step}"), (tokens, layer.K), wl.x_std)
        dY = gen.normal_bf16_bits(stream_seed(wl.seed, self._tag + f"/dY/{step}"), (tokens, layer.N), wl.dy_std)
        return X, dY


def _oracle_sample_step(O, wl, data, tokens, proxy_rows, step):
    """One oracle step of one layer shape on a bounded sample: `tokens` rows of
    X and dY through quantize / forward / dX / dB / dA, and `proxy_rows` rows
    of the proxy update.  Returns the two times (s)."""
    X, dY = data.rows(step, tokens)
    wq, s_w, K = data.wq, data.s_w, data.layer.K
    P = np.zeros((proxy_rows, K), dtype=np.float32)
    t0 = time.perf_counter()
    xq, s_x, _, _ = O.quantize(X)
    O.linear_fwd(xq, s_x, wq, s_w)
    dyq, s_dy, _, _ = O.quantize(dY)
    O.linear_dx(dyq, s_dy, wq, s_w)
    t64, _ = O.adapter_t(xq, s_x, data.A)
    db = O.adapter_db(dyq, s_dy, t64=t64)
    u64, _ = O.adapter_u(dyq, s_dy, data.B)
    O.adapter_da(xq, s_x, u64=u64)
    t1 = time.perf_counter()
    dB_inc = O.bf16_round(-wl.lr * O.bf16_to_f64(O.bf16_round(db)))
    O.proxy_update(np.ascontiguousarray(wq[:proxy_rows]), s_w, P, np.ascontiguousarray(dB_inc[:proxy_rows]),
                   data.A)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1


def _oracle_shapes(O, wl, r, n_stack):
    """(data, multiplicity) for every distinct layer shape of the workload."""
    seen = {}
    for layer in wl.layers:
        key = (layer.K, layer.N)
        if key not in seen:
            seen[key] = [_OracleData(O, wl, layer, r), 0]
        seen[key][1] += n_stack
    return list(seen.values())


def _sample_pass(O, wl, shapes, tokens, prows, step):
    """Runs the sample of every shape once; returns (seconds spent, the
    full-step seconds its per-token and per-row costs scale to)."""
    spent = full = 0.0
    for data, mult in shapes:
        tok = min(tokens, wl.M)
        pr = min(prows, data.layer.N)
        tg, tp = _oracle_sample_step(O, wl, data, tok, pr, step)
        spent += tg + tp
        full += mult * (tg * wl.M / tok + tp * data.layer.N / pr)
    return spent, full


def _sample_text(wl, shapes, tokens, prows, r):
    per = "; ".join(f"{d.layer.K}->{d.layer.N} x{m}: {min(prows, d.layer.N)} of {d.layer.N} proxy rows"
                    for d, m in shapes)
    return (f"per layer shape ({per}), r={r}: {min(tokens, wl.M)} of {wl.M} tokens through "
            f"quantize/fwd/dX/dB/dA and the proxy rows listed; the per-token and per-row costs are "
            f"scaled to one full step of every layer")


def cpu_baseline(wl, budget_s=20.0, r=None, n_stack=None):
    import oracle as O

    r = r or wl.r
    n_stack = n_stack or wl.n_stack
    cores = os.cpu_count() or 1
    O.set_threads(cores)
    shapes = _oracle_shapes(O, wl, r, n_stack)
    # a small probe sizes the sample to about budget_s seconds of CPU work
    tokens, prows = 64, 256
    spent, _ = _sample_pass(O, wl, shapes, tokens, prows, 0)
    scale = max(1.0, budget_s / max(spent, 1e-6))
    tokens, prows = int(tokens * scale), int(prows * scale)
    spent, full = _sample_pass(O, wl, shapes, tokens, prows, 1)
    return {"value": round(wl.M / full, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": _sample_text(wl, shapes, tokens, prows, r), "sample_seconds": round(spent, 3)}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return None, rank
    import oracle as O

    wl = WORKLOADS[args.workload]
    r = getattr(args, "rank", 0) or wl.r
    n_stack = getattr(args, "blocks", 0) or wl.n_stack
    cores = os.cpu_count() or 1
    O.set_threads(cores)
    shapes = _oracle_shapes(O, wl, r, n_stack)
    tokens, prows = 16, 64
    # size the per-step sample so the whole run stays within ~3 minutes
    spent, _ = _sample_pass(O, wl, shapes, tokens, prows, 0)
    budget = 150.0 / max(1, args.steps + args.warmup)
    scale = max(0.05, min(4.0, budget / max(spent, 1e-6)))
    tokens, prows = max(1, int(tokens * scale)), max(1, int(prows * scale))
    for i in range(args.warmup):
        _sample_pass(O, wl, shapes, tokens, prows, i)
    tot_spent = tot_full = 0.0
    for i in range(args.steps):
        sp, fu = _sample_pass(O, wl, shapes, tokens, prows, args.warmup + i)
        tot_spent += sp
        tot_full += fu
    full_step_s = tot_full / args.steps
    value = wl.M / full_step_s
    sample = _sample_text(wl, shapes, tokens, prows, r)
    layer0 = wl.layers[0]
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup,
        # what was timed: each step is the bounded sample, not a full step
        "ms_per_step": round(tot_spent / args.steps * 1e3, 3),
        "step": "a bounded sample of one step (see sample); value = the full step's tokens / the "
                "sample's per-token and per-row costs scaled to the full step",
        "full_step_ms_estimate": round(full_step_s * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": wl.name, "M": wl.M, "N": layer0.N, "K": layer0.K, "r": r,
                   "layers": len(wl.layers) * n_stack, "blocks": n_stack},
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
    ap.add_argument("--grouped", type=int, default=1,
                    help="forward GEMMs of layers that read one activation in one grouped launch (1) or not (0)")
    ap.add_argument("--e2e-outputs", type=int, default=0,
                    help="the e2e timing also copies every layer's Y and dX to the host (1) or reads back only "
                         "the step's metric (0)")
    ap.add_argument("--overlap-sgd", type=int, default=1,
                    help="run the caller's SGD on B on a second stream beside dX (1) or in line (0)")
    ap.add_argument("--proxy-defer", type=int, default=1,
                    help="carry the proxy clear of selected rows to the next step through row_mask (1) or "
                         "write it every step (0)")
    ap.add_argument("--proxy-tensor-from", type=int, default=256,
                    help="rank from which the proxy accumulates on the tensor cores (0: never)")
    ap.add_argument("--separate", type=int, default=1,
                    help="also time the separate bf16 and FP8 LoRA paths (the pages' comparison) (1) or not (0)")
    ap.add_argument("--topk", type=int, default=16,
                    help="also time the top-k proxy update merging this many of the r components (0: skip)")
    ap.add_argument("--rank", type=int, default=0, help="adapter rank (0: the workload's)")
    ap.add_argument("--blocks", type=int, default=0,
                    help="transformer blocks of a stacked workload (0: the workload's)")
    ap.add_argument("--slots", type=int, default=0,
                    help="input slots cycled by the timed steps (0: enough that their X and dY exceed "
                         "twice the 126 MB L2, at least 2)")
    ap.add_argument("--e2e", type=int, default=1, help="also time the step with host buffers (1) or skip it (0)")
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
