"""E5M2 gradients (C-15) on the GPU against the oracle: bit-exact codes and
scales from falqon_quantize_e5m2; dX (mixed E5M2 x E4M3 tcgen05 GEMM), dB and
dA from falqon_linear_bwd_e5m2 within the float tolerance (C-12); every
finite E5M2 code through the adapter products; infinity / NaN codes
propagated as the oracle propagates them."""

import os

import numpy as np
import pytest
import torch

import fp8_quantized_lora_b200 as F
import oracle as O
from gpu_util import dev_bf16, dev_f32, dev_u8, host, host_bf16_bits, status_word
from synthetic import gen

pytestmark = pytest.mark.gpu


def _quant_gpu(x_np):
    x = dev_bf16(x_np) if x_np.dtype == np.uint16 else dev_f32(x_np)
    st = status_word()
    codes, s, a = F.falqon_quantize(x, dev_status=st, fmt="e5m2")
    torch.cuda.synchronize()
    return host(codes), np.float32(host(s)[0]), np.float32(host(a)[0]), int(host(st)[0])


@pytest.mark.parametrize("shape,std,bf16", [
    ((256, 512), 1e-3, True),     # a gradient-like scale
    ((37, 48), 1.0, True),        # ragged
    ((1000, 1008), 1e-6, True),   # several chunks per CTA, tiny values
    ((300, 4096), 3.0, False),    # float32 input
    ((1, 16), 1.0, True),
])
def test_quantize_e5m2_bit_exact(cuda_device, shape, std, bf16):
    x = gen.normal_bf16_bits(41 + shape[0], shape, std) if bf16 else gen.normal_f32(41 + shape[0], shape, std)
    codes, s, a, st = _quant_gpu(x)
    rc, rs, ra, rst = O.quantize(x, "e5m2")
    assert st == rst == 0
    assert s.view(np.uint32) == rs.view(np.uint32) and a.view(np.uint32) == ra.view(np.uint32)
    np.testing.assert_array_equal(codes, rc)


def test_quantize_e5m2_nan_input_sets_status(cuda_device):
    x = gen.normal_f32(47, (64, 64), 1.0)
    x[3, 5] = np.nan
    codes, s, a, st = _quant_gpu(x)
    rc, rs, ra, rst = O.quantize(x, "e5m2")
    assert st == rst != 0
    np.testing.assert_array_equal(codes, rc)


def _bwd_gpu(dyq, s_dy, wq, s_w, xq, s_x, A, B, dx=True):
    st = status_word()
    dx_t, dA_t, dB_t = F.falqon_linear_bwd(dev_u8(dyq), dev_f32([s_dy]), dev_u8(wq), dev_f32([s_w]), dev_u8(xq),
                                           dev_f32([s_x]), dev_bf16(A), dev_bf16(B), dx=dx, dA=True, dB=True,
                                           dev_status=st, dy_fmt="e5m2")
    torch.cuda.synchronize()
    return ((host_bf16_bits(dx_t) if dx_t is not None else None), host_bf16_bits(dA_t), host_bf16_bits(dB_t),
            int(host(st)[0]))


def _oracle(dyq, s_dy, wq, s_w, xq, s_x, A, B):
    dx = O.linear_dx(dyq, s_dy, wq, s_w, dy_fmt="e5m2")
    t64, _ = O.adapter_t(xq, s_x, A)
    db = O.adapter_db(dyq, s_dy, t64=t64, dy_fmt="e5m2")
    u64, _ = O.adapter_u(dyq, s_dy, B, dy_fmt="e5m2")
    da = O.adapter_da(xq, s_x, u64=u64)
    return dx, da, db


def _case(seed, M, N, K, r):
    dyq, s_dy, _, _ = O.quantize(gen.normal_bf16_bits(seed, (M, N), 1e-3), "e5m2")
    wq, s_w, _, _ = O.quantize(gen.normal_f32(seed + 1, (N, K), 0.02))
    xq, s_x, _, _ = O.quantize(gen.normal_bf16_bits(seed + 2, (M, K), 1.0))
    A = gen.normal_bf16_bits(seed + 3, (r, K), 0.01)
    B = gen.normal_bf16_bits(seed + 4, (N, r), 0.01)
    return dyq, s_dy, wq, s_w, xq, s_x, A, B


@pytest.mark.parametrize("M,N,K,r", [
    (256, 512, 512, 16),
    (200, 272, 336, 32),     # ragged M, N, K
    (130, 256, 128, 64),
    (512, 256, 384, 80),
    (264, 256, 384, 512),    # large rank: the adapter products on the bf16 GEMM, E5M2 codes expanded
])
def test_backward_e5m2_matches_oracle(cuda_device, M, N, K, r):
    O.set_threads(os.cpu_count() or 8)
    case = _case(M + N + K + r, M, N, K, r)
    dx, da, db, st = _bwd_gpu(*case)
    rdx, rda, rdb = _oracle(*case)
    assert st == 0
    for g, ref, what in ((dx, rdx, "dX"), (da, rda, "dA"), (db, rdb, "dB")):
        rep = O.tolerance_report(g, ref)
        assert rep["ok"], (what, rep)


def test_every_e5m2_code_expands_exactly(cuda_device):
    """dYq cycles through every finite E5M2 code (subnormals, both zeros,
    +-57344); the adapter products must match the oracle."""
    M, N, K, r = 256, 384, 512, 32
    valid = np.array([c for c in range(256) if ((c >> 2) & 0x1F) != 31], dtype=np.uint8)
    dyq = valid[(np.arange(M * N) * 7 + 3) % valid.size].reshape(M, N)
    _, _, wq, s_w, xq, s_x, A, B = _case(61, M, N, K, r)
    s_dy = np.float32(4096.0)
    _, da, db, st = _bwd_gpu(dyq, s_dy, wq, s_w, xq, s_x, A, B, dx=None)
    _, rda, rdb = _oracle(dyq, s_dy, wq, s_w, xq, s_x, A, B)
    assert O.tolerance_report(db, rdb)["ok"]
    assert O.tolerance_report(da, rda)["ok"]


def test_infinity_and_nan_codes_propagate(cuda_device):
    """An infinity code and a NaN code in dYq go through the hardware
    conversion; the non-finite pattern of dB and dA matches the oracle's."""
    M, N, K, r = 128, 256, 256, 16
    dyq, s_dy, wq, s_w, xq, s_x, A, B = _case(67, M, N, K, r)
    dyq = dyq.copy()
    dyq[5, 77] = 0x7C    # +infinity
    dyq[9, 130] = 0xFF   # NaN
    _, da, db, _ = _bwd_gpu(dyq, s_dy, wq, s_w, xq, s_x, A, B, dx=None)
    _, rda, rdb = _oracle(dyq, s_dy, wq, s_w, xq, s_x, A, B)

    def nonfinite(bits):
        return (bits & 0x7F80) == 0x7F80

    assert np.array_equal(nonfinite(db), ~np.isfinite(rdb)) and (~np.isfinite(rdb)).any()
    assert np.array_equal(nonfinite(da), ~np.isfinite(rda)) and (~np.isfinite(rda)).any()
