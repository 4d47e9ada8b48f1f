"""Pins for the oracle's forward, dX and adapter-gradient products (C-5 .. C-8).

Independent references: exact rational arithmetic (fractions) on tiny
shapes, torch autograd in float64 for the LoRA gradient formulas (FALQON
rebuttal to reviewer 4, Q1: dL/dA = B^T dL/dO x^T, and the gradient of B from
the pre-computable A x), and special cases with closed forms.  Shapes are
chosen with M, N, K and r all different so a transposed operand cannot pass.
"""

from fractions import Fraction

import numpy as np
import torch

import oracle as O
from synthetic import gen

DEC = np.array([O.e4m3_decode(c) for c in range(256)])


def _codes(seed, shape):
    """Random finite E4M3 codes (NaN codes excluded)."""
    c = (gen.splitmix64(seed, int(np.prod(shape))) & np.uint64(0xFF)).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x38
    return c.reshape(shape)


def _bf16(seed, shape, std):
    return gen.normal_bf16_bits(seed, shape, std)


def _f(bits):
    return gen.bf16_bits_to_f32(bits).astype(np.float64)


def test_fwd_exact_rational_tiny():
    M, N, K = 3, 5, 7
    xq, wq = _codes(1, (M, K)), _codes(2, (N, K))
    s_x, s_w = np.float32(3.7), np.float32(0.11)
    y = O.linear_fwd(xq, s_x, wq, s_w)
    for m in range(M):
        for n in range(N):
            acc = sum(Fraction(DEC[xq[m, k]]) * Fraction(DEC[wq[n, k]]) for k in range(K))
            ref = acc / (Fraction(float(s_x)) * Fraction(float(s_w)))
            assert y[m, n] == float(ref)  # float() rounds the exact rational once


def test_fwd_matches_numpy_matmul_of_dequantized():
    M, N, K = 33, 48, 80
    xq, wq = _codes(3, (M, K)), _codes(4, (N, K))
    s_x, s_w = np.float32(20.5), np.float32(900.0)
    y = O.linear_fwd(xq, s_x, wq, s_w)
    ref = (DEC[xq] / np.float64(s_x)) @ (DEC[wq] / np.float64(s_w)).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_fwd_identity_backbone_returns_dequantized_x():
    M, K = 9, 32
    xq = _codes(5, (M, K))
    wq = np.zeros((K, K), dtype=np.uint8)
    np.fill_diagonal(wq, 0x38)  # code for 1.0
    s_x = np.float32(13.0)
    y = O.linear_fwd(xq, s_x, wq, np.float32(1.0))
    assert np.array_equal(y, DEC[xq] / np.float64(s_x))


def test_fwd_row_range_equals_full():
    xq, wq = _codes(6, (20, 48)), _codes(7, (16, 48))
    full = O.linear_fwd(xq, 2.0, wq, 3.0)
    part = O.linear_fwd(xq, 2.0, wq, 3.0, rows=(5, 13))
    assert np.array_equal(full[5:13], part)


def test_dx_is_forward_with_transposed_backbone():
    M, N, K = 11, 24, 40
    dyq, wq = _codes(8, (M, N)), _codes(9, (N, K))
    s_dy, s_w = np.float32(5000.0), np.float32(17.0)
    dx = O.linear_dx(dyq, s_dy, wq, s_w)
    assert np.array_equal(dx, O.linear_fwd(dyq, s_dy, np.ascontiguousarray(wq.T), s_w))


def test_dx_exact_rational_tiny():
    M, N, K = 2, 6, 4
    dyq, wq = _codes(10, (M, N)), _codes(11, (N, K))
    s_dy, s_w = np.float32(0.3), np.float32(7.0)
    dx = O.linear_dx(dyq, s_dy, wq, s_w)
    for m in range(M):
        for k in range(K):
            acc = sum(Fraction(DEC[dyq[m, n]]) * Fraction(DEC[wq[n, k]]) for n in range(N))
            assert dx[m, k] == float(acc / (Fraction(float(s_dy)) * Fraction(float(s_w))))


def _lora_case(seed, M=13, N=24, K=40, r=8):
    xq, dyq, wq = _codes(seed, (M, K)), _codes(seed + 1, (M, N)), _codes(seed + 2, (N, K))
    A = _bf16(seed + 3, (r, K), 0.05)
    B = _bf16(seed + 4, (N, r), 0.05)
    return xq, dyq, wq, A, B, np.float32(4.0), np.float32(300.0), np.float32(9.0)


def test_adapter_gradients_match_autograd_float64():
    # For O = X (W + B A)^T and L = <O, dY>: dL/dB = dY^T (X A^T), dL/dA = B^T dY^T X,
    # dL/dX = dY (W + B A).  Intermediates kept in float64 here (no bf16 rounding).
    xq, dyq, wq, A, B, s_x, s_dy, s_w = _lora_case(20)
    Xd = torch.tensor(DEC[xq] / np.float64(s_x), requires_grad=True)
    dYd = torch.tensor(DEC[dyq] / np.float64(s_dy))
    Wd = torch.tensor(DEC[wq] / np.float64(s_w))
    At = torch.tensor(_f(A), requires_grad=True)
    Bt = torch.tensor(_f(B), requires_grad=True)
    out = Xd @ (Wd + Bt @ At).T
    (out * dYd).sum().backward()
    t64, _ = O.adapter_t(xq, s_x, A)
    u64, _ = O.adapter_u(dyq, s_dy, B)
    db = O.adapter_db(dyq, s_dy, t64=t64)
    da = O.adapter_da(xq, s_x, u64=u64)
    assert np.allclose(db, Bt.grad.numpy(), rtol=1e-12, atol=1e-14)
    assert np.allclose(da, At.grad.numpy(), rtol=1e-12, atol=1e-14)
    # the backbone-only dX of the melded layer is the gradient through W alone
    Xd2 = torch.tensor(DEC[xq] / np.float64(s_x), requires_grad=True)
    ((Xd2 @ Wd.T) * dYd).sum().backward()
    dx = O.linear_dx(dyq, s_dy, wq, s_w)
    assert np.allclose(dx, Xd2.grad.numpy(), rtol=1e-12, atol=1e-14)


def test_adapter_t_u_exact_rational_and_bf16_rounding():
    xq, dyq, wq, A, B, s_x, s_dy, _ = _lora_case(30, M=3, N=5, K=6, r=2)
    t64, t16 = O.adapter_t(xq, s_x, A)
    u64, u16 = O.adapter_u(dyq, s_dy, B)
    Af, Bf = _f(A), _f(B)
    for m in range(3):
        for i in range(2):
            acc = sum(Fraction(DEC[xq[m, k]]) * Fraction(Af[i, k]) for k in range(6))
            assert t64[m, i] == float(acc / Fraction(float(s_x)))
            acc = sum(Fraction(DEC[dyq[m, n]]) * Fraction(Bf[n, i]) for n in range(5))
            assert u64[m, i] == float(acc / Fraction(float(s_dy)))
    assert np.array_equal(t16, O.bf16_round(t64))
    assert np.array_equal(u16, O.bf16_round(u64))


def test_db_and_da_match_numpy_products_of_exact_intermediates():
    xq, dyq, wq, A, B, s_x, s_dy, _ = _lora_case(40)
    t64, _ = O.adapter_t(xq, s_x, A)
    u64, _ = O.adapter_u(dyq, s_dy, B)
    db = O.adapter_db(dyq, s_dy, t64=t64)
    da = O.adapter_da(xq, s_x, u64=u64)
    ref_t = (DEC[xq] @ _f(A).T) / np.float64(s_x)
    ref_u = (DEC[dyq] @ _f(B)) / np.float64(s_dy)
    assert np.allclose(t64, ref_t, rtol=1e-13, atol=1e-16)
    assert np.allclose(u64, ref_u, rtol=1e-13, atol=1e-16)
    ref_db = (DEC[dyq].T @ ref_t) / np.float64(s_dy)
    ref_da = (ref_u.T @ DEC[xq]) / np.float64(s_x)
    assert np.allclose(db, ref_db, rtol=1e-12, atol=1e-15)
    assert np.allclose(da, ref_da, rtol=1e-12, atol=1e-15)
    # the bf16-rounded intermediates the oracle also reports are single roundings of T, U
    _, t16 = O.adapter_t(xq, s_x, A)
    assert np.array_equal(t16, O.bf16_round(t64))


def test_zero_b_gives_exactly_zero_u_and_da():
    xq, dyq, wq, A, _, s_x, s_dy, _ = _lora_case(50)
    B0 = np.zeros((24, 8), dtype=np.uint16)
    u64, u16 = O.adapter_u(dyq, s_dy, B0)
    assert np.all(u64 == 0) and np.all(u16 & 0x7FFF == 0)
    assert np.all(O.adapter_da(xq, s_x, u64=u64) == 0)


def test_zero_dy_gives_exactly_zero_db_and_dx():
    xq, _, wq, A, _, s_x, s_dy, s_w = _lora_case(60)
    dyq0 = np.zeros((13, 24), dtype=np.uint8)
    t64, _ = O.adapter_t(xq, s_x, A)
    assert np.all(O.adapter_db(dyq0, s_dy, t64=t64) == 0)
    assert np.all(O.linear_dx(dyq0, s_dy, wq, s_w) == 0)


def test_t_is_linear_in_a_under_power_of_two_scaling():
    xq, _, _, A, _, s_x, _, _ = _lora_case(70)
    A2 = gen.f32_to_bf16_bits(gen.bf16_bits_to_f32(A) * np.float32(2.0))
    t64a, t16a = O.adapter_t(xq, s_x, A)
    t64b, t16b = O.adapter_t(xq, s_x, A2)
    assert np.array_equal(t64b, 2 * t64a)
    assert np.array_equal(_f(t16b), 2 * _f(t16a))
