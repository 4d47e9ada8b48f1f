"""Folded quantized adapters on the GPU against the oracle (C-16).

A and B are quantized by falqon_quantize (codes and scales bit-exact against
the oracle); the forward and dX GEMMs then carry the adapter columns T and U,
and dB / dA are computed from them.  Y and dX must be bit-identical to the
unfolded GEMMs (the backbone tiles run the same MMAs in the same order); dB
and dA follow the float rule of oracle/tolerance.py against the oracle's
exact values; T, an intermediate held as a bf16 hi/lo pair, is checked
against the oracle's exact T to 2^-12 of its scale.
"""

import os

import numpy as np
import pytest
import torch

import fp8_quantized_lora_b200 as F
import oracle as O
from gpu_util import dev_bf16, dev_f32, dev_u8, host, host_bf16_bits, status_word
from synthetic import gen

pytestmark = pytest.mark.gpu


def _case(seed, M, N, K, r, b_std=1e-3):
    xq, s_x, _, _ = O.quantize(gen.normal_bf16_bits(seed, (M, K), 1.0))
    dyq, s_dy, _, _ = O.quantize(gen.normal_bf16_bits(seed + 1, (M, N), 1e-3))
    wq, s_w, _, _ = O.quantize(gen.normal_f32(seed + 2, (N, K), 0.02))
    A = gen.normal_bf16_bits(seed + 3, (r, K), 0.01)
    B = gen.normal_bf16_bits(seed + 4, (N, r), b_std) if b_std else np.zeros((N, r), np.uint16)
    return xq, s_x, dyq, s_dy, wq, s_w, A, B


def _run(xq, s_x, dyq, s_dy, wq, s_w, A, B, dx=True, dA=True, dB=True):
    st = status_word()
    aq, s_a, _ = F.falqon_quantize(dev_bf16(A), dev_status=st)
    bq, s_b, _ = F.falqon_quantize(dev_bf16(B), dev_status=st)
    X, Wd, DY = dev_u8(xq), dev_u8(wq), dev_u8(dyq)
    sx, sw, sdy = dev_f32([s_x]), dev_f32([s_w]), dev_f32([s_dy])
    y, t_saved = F.falqon_linear_fwd_folded(X, sx, Wd, sw, aq, s_a, dev_status=st)
    gdx, gdA, gdB = F.falqon_linear_bwd_folded(DY, sdy, Wd, sw, bq, s_b, X, sx, t_saved, A.shape[0],
                                               dx=dx, dA=dA, dB=dB, dev_status=st)
    y_plain = F.falqon_linear_fwd(X, sx, Wd, sw, dev_status=st)
    dx_plain, _, _ = F.falqon_linear_bwd(DY, sdy, Wd, sw, None, None, None, None, dx=True, dA=None, dB=None,
                                         dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    hi, lo = F.folded_t_planes(t_saved, xq.shape[0], A.shape[0])
    T = (hi.float() + lo.float()).t()[: xq.shape[0]].double().cpu().numpy()
    return dict(aq=host(aq), s_a=host(s_a)[0], bq=host(bq), s_b=host(s_b)[0], y=y, y_plain=y_plain,
                dx=gdx, dx_plain=dx_plain, dA=gdA, dB=gdB, T=T)


def _check(case, g, want_da=True):
    xq, s_x, dyq, s_dy, wq, s_w, A, B = case
    raq, rs_a, _, _ = O.quantize(A)
    rbq, rs_b, _, _ = O.quantize(B)
    assert np.array_equal(g["aq"], raq) and g["s_a"].view(np.uint32) == rs_a.view(np.uint32)
    assert np.array_equal(g["bq"], rbq) and g["s_b"].view(np.uint32) == rs_b.view(np.uint32)
    assert torch.equal(g["y"].view(torch.int16), g["y_plain"].view(torch.int16))
    if g["dx"] is not None:
        assert torch.equal(g["dx"].view(torch.int16), g["dx_plain"].view(torch.int16))
    t64, db, u64, da = O.folded_adapter_grads(xq, s_x, dyq, s_dy, raq, rs_a, rbq, rs_b)
    scale = np.abs(t64).max()
    np.testing.assert_allclose(g["T"], t64, rtol=2 ** -12, atol=2 ** -12 * scale)
    if g["dB"] is not None:
        rep = O.tolerance_report(host_bf16_bits(g["dB"]), db)
        assert rep["ok"], ("dB", rep)
    if want_da and g["dA"] is not None:
        rep = O.tolerance_report(host_bf16_bits(g["dA"]), da)
        assert rep["ok"], ("dA", rep)
    return t64, db, u64, da


CASES = [
    (256, 512, 512, 16),     # the tiny parity workload's shapes
    (200, 272, 336, 32),     # ragged M, N, K
    (130, 128, 192, 64),     # one row past a tile
    (512, 256, 384, 80),     # r not a power of two
    (128, 256, 512, 320),    # two adapter tiles (r > 256)
    (3, 256, 512, 16),       # fewer tokens than a tile
    (1000, 4096, 1024, 64),  # many backbone tiles beside one adapter tile
]


@pytest.mark.parametrize("M,N,K,r", CASES)
def test_folded_step_matches_oracle(cuda_device, M, N, K, r):
    O.set_threads(os.cpu_count() or 8)
    case = _case(M + N + K + r, M, N, K, r)
    _check(case, _run(*case))


def test_zero_b_gives_exactly_zero_da(cuda_device):
    case = _case(5, 256, 512, 512, 16, b_std=0)
    g = _run(*case)
    _check(case, g)
    assert not torch.any(g["dA"].float() != 0)


def test_adapter_columns_without_the_backbone_outputs(cuda_device):
    """dX not requested: the dX GEMM runs the U tiles alone; dB alone skips U."""
    O.set_threads(os.cpu_count() or 8)
    case = _case(11, 384, 256, 512, 32)
    g = _run(*case, dx=None)
    assert g["dx"] is None
    _check(case, g)
    g2 = _run(*case, dx=None, dA=None)
    assert g2["dA"] is None
    _check(case, g2, want_da=False)


def test_llama_attention_full_size(cuda_device):
    """The attention projection at full size: Y and dX bit-identical to the
    unfolded GEMMs; dB and dA on sampled ranks, every row / column of them."""
    from synthetic.workloads import WORKLOADS, layer_inputs

    O.set_threads(os.cpu_count() or 8)
    wl = WORKLOADS["llama7b_attn_proj_4096x4096x4096_r64"]
    d = layer_inputs(wl, wl.layers[0], with_b=True)
    xq, s_x, _, _ = O.quantize(d["X"])
    dyq, s_dy, _, _ = O.quantize(d["dY"])
    wq, s_w, _, _ = O.quantize(d["W"])
    g = _run(xq, s_x, dyq, s_dy, wq, s_w, d["A"], d["B"])
    assert torch.equal(g["y"].view(torch.int16), g["y_plain"].view(torch.int16))
    assert torch.equal(g["dx"].view(torch.int16), g["dx_plain"].view(torch.int16))
    raq, rs_a, _, _ = O.quantize(d["A"])
    rbq, rs_b, _, _ = O.quantize(d["B"])
    assert np.array_equal(g["aq"], raq) and np.array_equal(g["bq"], rbq)
    ranks = [0, 1, 31, 63]
    t64 = O.folded_t(xq, s_x, raq[ranks], rs_a)
    np.testing.assert_allclose(g["T"][:, ranks], t64, rtol=2 ** -12, atol=2 ** -12 * np.abs(t64).max())
    rep = O.tolerance_report(host_bf16_bits(g["dB"])[:, ranks], O.adapter_db(dyq, s_dy, t64=t64))
    assert rep["ok"], ("dB", rep)
    u64 = O.folded_u(dyq, s_dy, np.ascontiguousarray(rbq[:, ranks]), rs_b)
    rep = O.tolerance_report(host_bf16_bits(g["dA"])[ranks, :], O.adapter_da(xq, s_x, u64=u64))
    assert rep["ok"], ("dA", rep)
