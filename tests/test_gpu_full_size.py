"""Every workload of the step at full size, one whole step through the C ABI
in the call sequence the benchmark times (quantize W once; quantize X, the
forward GEMM, quantize dY, the backward with dX, dA and dB, the caller's SGD
increment, the proxy update).  The oracle checks:

  - every code and scale of W, X and dY (bit-exact, whole tensors);
  - Y and dX on rows that touch every 1024-row group and the last row;
  - dB and dA on a sample of ranks, every row of dB and every column of dA
    for those ranks (the float rule of oracle/tolerance.py, with its floor
    taken over the sample, which is never looser than over the tensor);
  - the proxy update on a sample of rows (bit-exact codes, proxy and row
    mask; rows are independent, so the oracle runs on those rows alone,
    from the GPU's own dB increment); the selected count equals the mask's
    sum.

The rank sweep runs the attention shape at r = 256 .. 8192: the adapter
products then span many rank tiles and the proxy's float32 FMA chains run
8192 terms.
"""

import os

import numpy as np
import pytest
import torch

import fp8_quantized_lora_b200 as F
import oracle as O
from gpu_util import dev_bf16, dev_f32, host, host_bf16_bits, sample_rows, status_word
from synthetic.workloads import WORKLOADS, layer_inputs

pytestmark = pytest.mark.gpu

CASES = [
    ("llama7b_attn_proj_4096x4096x4096_r64", "proj", 0, None),
    ("llama7b_mlp_8192tok_r64", "gate", 0, None),
    ("llama7b_mlp_8192tok_r64", "down", 0, None),
    ("llama2_7b_stack_32x7_4096tok_r16", "q", 0, None),
    ("llama2_7b_stack_32x7_4096tok_r16", "down", 31, None),
    ("rank_sweep_4096cube", "proj", 0, 256),
    ("rank_sweep_4096cube", "proj", 0, 1024),
    ("rank_sweep_4096cube", "proj", 0, 4096),
    ("rank_sweep_4096cube", "proj", 0, 8192),
]


def _ids(c):
    return f"{c[0]}-{c[1]}-b{c[2]}" + (f"-r{c[3]}" if c[3] else "")


def _close(G, R, what):
    rep = O.tolerance_report(G, R)
    assert rep["ok"], (what, rep)


@pytest.mark.parametrize("name,layer,block,rank", CASES, ids=[_ids(c) for c in CASES])
def test_full_step_sampled(cuda_device, name, layer, block, rank):
    O.set_threads(os.cpu_count() or 8)
    wl = WORKLOADS[name]
    lay = next(x for x in wl.layers if x.name == layer)
    r = rank or wl.r
    d = layer_inputs(wl, lay, block=block, r=r, with_b=True)
    M, N, K = wl.M, lay.N, lay.K
    # an increment that selects part of the rows at step 0 (P starts at zero)
    lr = 1e-4 * (64.0 / r) ** 0.5

    st = status_word()
    wq, s_w, _ = F.falqon_quantize(dev_f32(d["W"]), dev_status=st)
    xq, s_x, _ = F.falqon_quantize(dev_bf16(d["X"]), dev_status=st)
    y = F.falqon_linear_fwd(xq, s_x, wq, s_w, dev_status=st)
    dyq, s_dy, _ = F.falqon_quantize(dev_bf16(d["dY"]), dev_status=st)
    A, B = dev_bf16(d["A"]), dev_bf16(d["B"])
    dx, dA, dB = F.falqon_linear_bwd(dyq, s_dy, wq, s_w, xq, s_x, A, B, dev_status=st)
    dB_inc = torch.mul(dB, -lr)  # the caller's SGD increment, bf16
    wq0 = host(wq).copy()
    P = torch.zeros((N, K), dtype=torch.float32, device=wq.device)
    mask, cnt = F.falqon_proxy_update(wq, s_w, P, dB_inc, A, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0

    # quantize: whole tensors, bit-exact
    rw, rs_w, _, _ = O.quantize(d["W"])
    rx, rs_x, _, _ = O.quantize(d["X"])
    rdy, rs_dy, _, _ = O.quantize(d["dY"])
    for what, g, ref in (("Wq", wq0, rw), ("Xq", host(xq), rx), ("dYq", host(dyq), rdy)):
        assert np.array_equal(g, ref), what
    for what, g, ref in (("s_W", s_w, rs_w), ("s_X", s_x, rs_x), ("s_dY", s_dy, rs_dy)):
        assert host(g)[0].view(np.uint32) == np.float32(ref).view(np.uint32), what

    # forward and dX: sampled rows
    yb, dxb = host_bf16_bits(y), host_bf16_bits(dx)
    for m in sample_rows(M, 1024):
        _close(yb[m], O.linear_fwd(rx, rs_x, rw, rs_w, rows=(m, m + 1))[0], ("Y", m))
        _close(dxb[m], O.linear_dx(rdy, rs_dy, rw, rs_w, rows=(m, m + 1))[0], ("dX", m))

    # dB and dA: sampled ranks (first, second, middle, last)
    ranks = sorted({0, 1, r // 2, r - 1})
    t64, _ = O.adapter_t(rx, rs_x, d["A"][ranks])
    _close(host_bf16_bits(dB)[:, ranks], O.adapter_db(rdy, rs_dy, t64=t64), "dB")
    u64, _ = O.adapter_u(rdy, rs_dy, d["B"][:, ranks])
    _close(host_bf16_bits(dA)[ranks, :], O.adapter_da(rx, rs_x, u64=u64), "dA")

    # proxy update: sampled rows from the GPU's increment
    rows = sample_rows(N, 256)
    inc = host_bf16_bits(dB_inc)
    rwq, rP, rmask, rcnt = O.proxy_update(rw[rows], rs_w, np.zeros((len(rows), K), np.float32),
                                          inc[rows], d["A"])
    gm = host(mask)
    assert np.array_equal(host(wq)[rows], rwq)
    assert np.array_equal(host(P)[rows].view(np.uint32), rP.view(np.uint32))
    assert np.array_equal(gm[rows], rmask)
    assert int(host(cnt)[0]) == int(gm.sum())
    # rows outside the mask keep their codes
    keep = gm == 0
    assert np.array_equal(host(wq)[keep], wq0[keep])
