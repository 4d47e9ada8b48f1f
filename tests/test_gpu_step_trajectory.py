"""One hundred training steps of the tiny workload on the GPU, checked step by
step against the oracle.

At every step the oracle starts from the GPU's state after the previous step
(Wq, P and B), takes that step's fresh X and dY, and must reproduce the
step: codes and scales bit-exact, Y, dX, dB and dA within the float rule of
oracle/tolerance.py, and the proxy update (fed the GPU's own SGD increment)
bit-exact.  Trajectories of two implementations can part through a single
boundary flip, so the per-step comparison is the well-defined one.
"""

import numpy as np
import pytest
import torch

import fp8_quantized_lora_b200 as F
import oracle as O
from gpu_util import dev_bf16, dev_f32, host, host_bf16_bits, status_word
from oracle.step import layer_step
from synthetic.workloads import WORKLOADS, layer_inputs

pytestmark = pytest.mark.gpu

STEPS = 100


def _close(G, R, what):
    rep = O.tolerance_report(G, R)
    assert rep["ok"], (what, rep)


def test_tiny_workload_hundred_steps_stepwise(cuda_device):
    wl = WORKLOADS["tiny_256x512x512_r16"]
    lay = wl.layers[0]
    d0 = layer_inputs(wl, lay, step=0)
    st = status_word()
    wq, s_w, _ = F.falqon_quantize(dev_f32(d0["W"]), dev_status=st)
    A = dev_bf16(d0["A"])
    B = dev_bf16(d0["B"])  # zero at step 0
    P = torch.zeros((lay.N, lay.K), dtype=torch.float32, device=wq.device)
    rw, rs_w, _, _ = O.quantize(d0["W"])
    torch.cuda.synchronize()
    assert np.array_equal(host(wq), rw) and host(s_w)[0] == rs_w
    selected = []
    for t in range(STEPS):
        d = layer_inputs(wl, lay, step=t)
        pre_wq, pre_P, pre_B = host(wq).copy(), host(P).copy(), host_bf16_bits(B).copy()
        # the GPU step, in the benchmark's call order
        xq, s_x, _ = F.falqon_quantize(dev_bf16(d["X"]), dev_status=st)
        y = F.falqon_linear_fwd(xq, s_x, wq, s_w, dev_status=st)
        dyq, s_dy, _ = F.falqon_quantize(dev_bf16(d["dY"]), dev_status=st)
        dx, dA, dB = F.falqon_linear_bwd(dyq, s_dy, wq, s_w, xq, s_x, A, B, dev_status=st)
        dB_inc = torch.mul(dB, -wl.lr)  # the caller's SGD step on B
        B.add_(dB_inc)
        mask, cnt = F.falqon_proxy_update(wq, s_w, P, dB_inc, A, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0, t
        # the oracle, from the GPU's state before the step
        ref = layer_step(d["X"], pre_wq, rs_w, d0["A"], pre_B, d["dY"], pre_P,
                         dB_inc=host_bf16_bits(dB_inc))
        assert np.array_equal(host(xq), ref["xq"]) and host(s_x)[0] == ref["s_x"], t
        assert np.array_equal(host(dyq), ref["dyq"]) and host(s_dy)[0] == ref["s_dy"], t
        _close(host_bf16_bits(y), ref["y"], ("Y", t))
        _close(host_bf16_bits(dx), ref["dx"], ("dX", t))
        _close(host_bf16_bits(dB), ref["db"], ("dB", t))
        if t > 0:  # B = 0 at step 0 makes dA exactly zero (checked below)
            _close(host_bf16_bits(dA), ref["da"], ("dA", t))
        else:
            assert not torch.any(dA.float() != 0)
        assert np.array_equal(host(wq), ref["wq_new"]), t
        assert np.array_equal(host(P).view(np.uint32), ref["P_new"].view(np.uint32)), t
        assert np.array_equal(host(mask), ref["mask"]), t
        assert int(host(cnt)[0]) == ref["n_selected"], t
        selected.append(int(host(cnt)[0]))
    # the trajectory exercises the selection: rows are requantized along the way
    assert sum(selected) > 0
