"""Pins for the oracle's folded quantized adapters (C-16).

The folded path quantizes A and B like any other operand and reads their
products out of the backbone GEMMs.  References independent of the
composition in oracle/__init__.py:
  - adapters whose values are exactly E4M3 values times a power of two
    quantize losslessly, and then the folded T, U, dB and dA must equal the
    bf16-adapter path of C-7 / C-8 (separate C code, pinned elsewhere);
  - for arbitrary adapters, T and U differ from the bf16 path by no more
    than the triangle-inequality bound of the adapters' quantization errors;
  - a brute-force float64 product of decoded codes on a tiny case.
"""

import numpy as np

import oracle as O
from synthetic import gen

DEC = np.array([O.e4m3_decode(c) for c in range(256)])
FINITE = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)


def _exact_adapter(seed, shape, j):
    """bf16 bits of dec(c) * 2^-j for random finite codes c, one of them 448;
    returns (bits, codes)."""
    rng = np.random.default_rng(seed)
    c = rng.choice(FINITE, size=shape).astype(np.uint8)
    c.flat[rng.integers(c.size)] = 0x7E  # amax = 448 * 2^-j, so s = 2^j exactly
    vals = np.ldexp(DEC[c], -j).astype(np.float32)
    assert np.array_equal(vals.astype(np.float64), np.ldexp(DEC[c], -j))  # exact in f32 and bf16
    return gen.f32_to_bf16_bits(vals), c


def _bf16(bits):
    return gen.bf16_bits_to_f32(bits).astype(np.float64)


def test_lossless_adapters_reduce_to_the_bf16_adapter_path():
    M, N, K, r = 40, 48, 64, 16
    xq, s_x, _, _ = O.quantize(gen.normal_bf16_bits(1, (M, K), 1.0))
    dyq, s_dy, _, _ = O.quantize(gen.normal_bf16_bits(2, (M, N), 1e-3))
    A, ca = _exact_adapter(3, (r, K), 10)
    B, cb = _exact_adapter(4, (N, r), 14)
    aq, s_a, _, _ = O.quantize(A)
    bq, s_b, _, _ = O.quantize(B)
    # the quantization is lossless: codes and power-of-two scales come back
    assert s_a == np.float32(2.0 ** 10) and s_b == np.float32(2.0 ** 14)
    assert np.array_equal(DEC[aq], DEC[ca]) and np.array_equal(DEC[bq], DEC[cb])
    t64, db, u64, da = O.folded_adapter_grads(xq, s_x, dyq, s_dy, aq, s_a, bq, s_b)
    rt, _ = O.adapter_t(xq, s_x, A)
    ru, _ = O.adapter_u(dyq, s_dy, B)
    # every product of two E4M3 values is exact and K such sums fit float64's
    # mantissa, so both paths round only at the final division
    np.testing.assert_allclose(t64, rt, rtol=4e-16, atol=0)
    np.testing.assert_allclose(u64, ru, rtol=4e-16, atol=0)
    np.testing.assert_allclose(db, O.adapter_db(dyq, s_dy, t64=rt), rtol=1e-14, atol=1e-300)
    np.testing.assert_allclose(da, O.adapter_da(xq, s_x, u64=ru), rtol=1e-14, atol=1e-300)


def test_folded_products_are_within_the_adapter_quantization_error():
    M, N, K, r = 24, 32, 96, 16
    xq, s_x, _, _ = O.quantize(gen.normal_bf16_bits(5, (M, K), 1.0))
    dyq, s_dy, _, _ = O.quantize(gen.normal_bf16_bits(6, (M, N), 1e-3))
    A = gen.normal_bf16_bits(7, (r, K), 0.01)
    B = gen.normal_bf16_bits(8, (N, r), 1e-3)
    aq, s_a, _, _ = O.quantize(A)
    bq, s_b, _, _ = O.quantize(B)
    ea = np.abs(_bf16(A) - DEC[aq] / np.float64(s_a))  # per-element error of A~
    eb = np.abs(_bf16(B) - DEC[bq] / np.float64(s_b))
    X = np.abs(DEC[xq]) / np.float64(s_x)
    D = np.abs(DEC[dyq]) / np.float64(s_dy)
    t64 = O.folded_t(xq, s_x, aq, s_a)
    u64 = O.folded_u(dyq, s_dy, bq, s_b)
    rt, _ = O.adapter_t(xq, s_x, A)
    ru, _ = O.adapter_u(dyq, s_dy, B)
    assert np.all(np.abs(t64 - rt) <= X @ ea.T * (1 + 1e-12) + 1e-300)
    assert np.all(np.abs(u64 - ru) <= D @ eb * (1 + 1e-12) + 1e-300)
    # ... and the adapters were not lossless, so the bound is exercised
    assert np.abs(t64 - rt).max() > 0 and np.abs(u64 - ru).max() > 0


def test_brute_force_tiny():
    M, N, K, r = 3, 16, 16, 2
    xq, s_x, _, _ = O.quantize(gen.normal_bf16_bits(9, (M, K), 1.0))
    dyq, s_dy, _, _ = O.quantize(gen.normal_bf16_bits(10, (M, N), 1.0))
    aq, s_a, _, _ = O.quantize(gen.normal_bf16_bits(11, (r, K), 0.01))
    bq, s_b, _, _ = O.quantize(gen.normal_bf16_bits(12, (N, r), 0.01))
    T = np.zeros((M, r))
    U = np.zeros((M, r))
    for m in range(M):
        for i in range(r):
            T[m, i] = sum(DEC[xq[m, k]] * DEC[aq[i, k]] for k in range(K)) / (float(s_x) * float(s_a))
            U[m, i] = sum(DEC[dyq[m, n]] * DEC[bq[n, i]] for n in range(N)) / (float(s_dy) * float(s_b))
    t64, db, u64, da = O.folded_adapter_grads(xq, s_x, dyq, s_dy, aq, s_a, bq, s_b)
    np.testing.assert_allclose(t64, T, rtol=1e-13, atol=0)
    np.testing.assert_allclose(u64, U, rtol=1e-13, atol=0)
    dB = np.array([[sum(DEC[dyq[m, n]] / float(s_dy) * T[m, i] for m in range(M)) for i in range(r)]
                   for n in range(N)])
    dA = np.array([[sum(U[m, i] * DEC[xq[m, k]] / float(s_x) for m in range(M)) for k in range(K)]
                   for i in range(r)])
    np.testing.assert_allclose(db, dB, rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(da, dA, rtol=1e-12, atol=1e-300)


def test_without_b_only_t_and_db():
    xq, s_x, _, _ = O.quantize(gen.normal_bf16_bits(13, (8, 32), 1.0))
    dyq, s_dy, _, _ = O.quantize(gen.normal_bf16_bits(14, (8, 16), 1.0))
    aq, s_a, _, _ = O.quantize(gen.normal_bf16_bits(15, (4, 32), 0.01))
    t64, db, u64, da = O.folded_adapter_grads(xq, s_x, dyq, s_dy, aq, s_a)
    assert t64.shape == (8, 4) and db.shape == (16, 4) and u64 is None and da is None
