"""Pins for the oracle's E5M2 gradient format (C-15).

References independent of the oracle's code: numpy's IEEE binary16 decoding
(an E5M2 code is the high byte of a binary16 value with the same exponent
bias), a brute-force nearest-value search over every finite code (ties to
the even mantissa, saturating), and float64 matrix products of the decoded
codes for the steps that read dY."""

import numpy as np
import pytest

import oracle as O
from synthetic import gen


def _f16_decode(c):
    return np.array([np.uint16(int(x) << 8) for x in np.atleast_1d(c)], dtype=np.uint16).view(np.float16).astype(np.float64)


DEC5 = np.array([O.e5m2_decode(c) for c in range(256)])


def test_decode_matches_binary16_high_byte():
    ref = _f16_decode(np.arange(256))
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(DEC5), nan)
    assert np.array_equal(DEC5[~nan], ref[~nan])
    assert np.array_equal(np.signbit(DEC5[~nan]), np.signbit(ref[~nan]))
    assert DEC5[0x7B] == 57344.0 and DEC5[0x01] == 2.0 ** -16 and np.isinf(DEC5[0x7C])


def _brute(v):
    """Nearest finite E5M2 code by search; ties to the even mantissa; saturating."""
    finite = [c for c in range(256) if np.isfinite(DEC5[c])]
    vals = DEC5[finite]
    out = []
    for x in np.asarray(v, dtype=np.float32).ravel():
        x = np.float64(x)
        if np.isnan(x):
            out.append(0x7F)
            continue
        if abs(x) >= 57344.0:
            out.append(0xFB if np.signbit(x) else 0x7B)
            continue
        d = np.abs(vals - x)
        best = np.flatnonzero(d == d.min())
        cands = [finite[i] for i in best]
        same_sign = [c for c in cands if bool(c & 0x80) == bool(np.signbit(x))]
        cands = same_sign or cands
        if len(cands) > 1:  # a tie between neighbours: the even mantissa wins
            cands = [c for c in cands if (c & 1) == 0] or cands
        out.append(cands[0])
    return np.array(out, dtype=np.uint8).reshape(np.shape(v))


def test_encode_matches_brute_force_search():
    rng = np.random.default_rng(5)
    v = np.concatenate([
        rng.standard_normal(3000).astype(np.float32) * np.float32(10.0) ** rng.integers(-6, 5, 3000),
        (DEC5[4:0x7B][::3] * 1.0).astype(np.float32),                          # exact codes
        ((DEC5[4:0x7A] + DEC5[5:0x7B]) / 2).astype(np.float32),                 # exact halfway points
        np.array([0.0, -0.0, 2 ** -17, 3 * 2 ** -17, 60000, -1e30, np.inf, -np.inf], dtype=np.float32),
    ])
    got = O.e5m2_encode(v)
    ref = _brute(v)
    # zeros: the encoder keeps the sign of a value that rounds to zero
    assert np.array_equal(got, ref) or np.array_equal(got & 0x7F, ref & 0x7F)
    nz = DEC5[ref] != 0
    assert np.array_equal(got[nz], ref[nz])


def test_quantize_e5m2_scale_and_codes():
    x = gen.normal_f32(7, (64, 80), 3.0)
    codes, s, a, st = O.quantize(x, "e5m2")
    assert st == 0 and a == np.float32(np.abs(x).max())
    assert s == np.float32(np.float32(57344.0) / a)
    ref = _brute((x * s).astype(np.float32))
    assert np.array_equal(codes, ref)


def test_dx_and_adapter_products_read_e5m2():
    M, N, K, r = 24, 32, 48, 8
    dyq, s_dy, _, _ = O.quantize(gen.normal_f32(8, (M, N), 1.0), "e5m2")
    wq, s_w, _, _ = O.quantize(gen.normal_f32(9, (N, K), 0.02))
    B = gen.normal_bf16_bits(10, (N, r), 0.01)
    xq, s_x, _, _ = O.quantize(gen.normal_f32(11, (M, K), 1.0))
    A = gen.normal_bf16_bits(12, (r, K), 0.01)
    D = DEC5[dyq]
    W = np.array([O.e4m3_decode(c) for c in range(256)])[wq]
    dx = O.linear_dx(dyq, s_dy, wq, s_w, dy_fmt="e5m2")
    np.testing.assert_allclose(dx, D @ W / (np.float64(s_dy) * np.float64(s_w)), rtol=1e-12, atol=0)
    u64, _ = O.adapter_u(dyq, s_dy, B, dy_fmt="e5m2")
    Bf = O.bf16_to_f64(B)
    np.testing.assert_allclose(u64, D @ Bf / np.float64(s_dy), rtol=1e-12, atol=1e-300)
    t64, _ = O.adapter_t(xq, s_x, A)
    db = O.adapter_db(dyq, s_dy, t64=t64, dy_fmt="e5m2")
    np.testing.assert_allclose(db, D.T @ t64 / np.float64(s_dy), rtol=1e-12, atol=1e-300)
    # the E4M3 reading of the same bytes differs: the format argument is used
    assert not np.allclose(O.linear_dx(dyq, s_dy, wq, s_w), dx)
