"""bench.py's output contract, checked on the CPU through its reference arm
(the oracle timed on the host): one JSON line with the keys and types the
benchmark driver reads."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run(
        [sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3",
         "--workload", "tiny_256x512x512_r16"],
        cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1 and d["value"] > 0
    assert d["config"]["workload"] == "tiny_256x512x512_r16"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0


def test_warmup_below_three_is_refused():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1"],
                         cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert out.returncode != 0 and "warmup" in out.stderr


def test_phase_work_matches_the_stated_algorithmic_work():
    """The roofline numerators bench.py divides by the measured times: the
    per-step work stated for each kernel, recomputed by hand for the
    attention projection (M = N = K = 4096, r = 64) and a rank-16 layer."""
    import types

    sys.path.insert(0, ROOT)
    import bench

    st = types.SimpleNamespace(M=4096, N=4096, K=4096, r=64)
    w = bench._phase_work(st)
    M = N = K = 4096
    assert w["fwd"]["flops"] == 2 * M * N * K == 137438953472
    assert w["dX"]["flops"] == w["fwd"]["flops"]
    assert w["fwd"]["bytes"] == M * K + N * K + 2 * M * N  # codes in, bf16 out
    assert w["quantX"]["bytes"] == 3 * M * K  # bf16 in, codes out
    assert w["quantdY"]["bytes"] == 3 * M * N
    assert w["adapters"]["flops"] == 4 * M * 64 * (N + K)  # T, U, dB, dA
    assert w["proxy"]["flops"] == 2 * N * K * 64  # r FMAs per element
    assert w["proxy"]["bytes"] == 9 * N * K + 2 * 64 * (N + K)  # read P and Wq, write P; the adapters
    # at r = 64 the FMA chain outlasts the 9 bytes per element; at r = 16 HBM bounds it
    assert w["proxy"]["bound"] == "alu"
    assert bench._phase_work(types.SimpleNamespace(M=4096, N=4096, K=4096, r=16))["proxy"]["bound"] == "hbm"
    assert w["fwd"]["bound"] == w["dX"]["bound"] == "tensor" and w["quantX"]["bound"] == "hbm"


def test_traffic_is_withheld_when_a_source_changes(tmp_path, monkeypatch):
    """bench.py reports a captured DRAM traffic figure only while the kernel
    sources hash as they did at the capture; every committed figure matches
    the committed sources."""
    import hashlib
    import types

    sys.path.insert(0, ROOT)
    import bench

    def step(t):
        return types.SimpleNamespace(wl=types.SimpleNamespace(name=t["workload"]), r=t["r"],
                                     defer_clear=t["defer_clear"])

    for phase, t in bench.TRAFFIC.items():  # committed figures are current
        assert t["workload"] in bench.WORKLOADS, phase
        assert bench._traffic(phase, step(t)) == t["bytes"], phase
        assert "ncu" in t["capture"] and "--clock-control none" in t["capture"]
    src = tmp_path / "k.cu"
    src.write_text("kernel")
    entry = {"workload": "w", "r": 64, "defer_clear": True, "bytes": 123, "capture": "ncu --clock-control none ...",
             "sources": {"k.cu": hashlib.sha256(b"kernel").hexdigest()}}
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "TRAFFIC", {"proxy": entry})
    assert bench._traffic("proxy", step(entry)) == 123
    # another workload, rank or clear mode than the capture's: no figure
    assert bench._traffic("proxy", step(dict(entry, workload="v"))) is None
    assert bench._traffic("proxy", step(dict(entry, r=16))) is None
    assert bench._traffic("proxy", step(dict(entry, defer_clear=False))) is None
    src.write_text("changed")
    assert bench._traffic("proxy", step(entry)) is None
    assert bench._traffic("fwd", step(entry)) is None  # no capture recorded for it


def test_step_work_counts_each_activation_group_once():
    """Whole-step work of the MLP workload (gate and up read the same X):
    quantize X is counted once per activation group, every other phase once
    per layer, so that a shared input's bytes are not counted twice."""
    import types

    sys.path.insert(0, ROOT)
    import bench
    from synthetic import WORKLOADS

    wl = WORKLOADS["llama7b_mlp_8192tok_r64"]
    M, r = wl.M, wl.r
    layers = [types.SimpleNamespace(N=l.N, K=l.K) for l in wl.layers]
    groups = {}
    for l in wl.layers:
        groups.setdefault((0, l.x_group), l.K)
    st = types.SimpleNamespace(M=M, r=r, layers=layers, groups=groups,
                               calls_per_step={p: 1 for p in bench.Step.PHASES})
    w = bench._step_work(st)
    assert len(groups) == 2 and len(layers) == 3
    assert w["quantX"]["bytes"] == 3 * M * (4096 + 11008)             # x_mlp once, x_down once
    assert w["quantdY"]["bytes"] == 3 * M * (11008 + 11008 + 4096)    # every layer's dY
    assert w["fwd"]["flops"] == w["dX"]["flops"] == 2 * M * 3 * 4096 * 11008
    assert w["proxy"]["flops"] == 2 * r * 3 * 4096 * 11008
    assert w["adapters"]["flops"] == 4 * M * r * (3 * (4096 + 11008))
