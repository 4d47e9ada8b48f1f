"""Pins for the oracle's separate LoRA paths (C-17), the comparison the
rank sweep measures.

References independent of the composition under test:
  - the unrounded bf16 path against float64 automatic differentiation of the
    separate-adapter layer (pins every operand role and transpose);
  - the float64 product against a brute-force Python loop;
  - zero adapters, which reduce every output to the backbone's or to zero;
  - the FP8 path equal to the bf16 path, bit for bit, on inputs whose every
    quantization is lossless (values on the E4M3 grid times powers of two,
    with the tensor's largest value planted so the scale is a power of two);
  - the FP8 products against brute-force loops over decoded codes.
"""

import numpy as np
import pytest

import oracle as O
from oracle import separate as SP
from synthetic import gen

DEC = np.array([O.e4m3_decode(c) for c in range(256)])


def _bf16(x):
    return gen.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _case(seed, M=24, N=32, K=48, r=16):
    X = gen.normal_bf16_bits(seed, (M, K), 1.0)
    W = gen.normal_f32(seed + 1, (N, K), 0.02)
    A = gen.normal_bf16_bits(seed + 2, (r, K), 0.01)
    B = gen.normal_bf16_bits(seed + 3, (N, r), 0.01)
    dY = gen.normal_bf16_bits(seed + 4, (M, N), 1e-3)
    wq, s_w, _, _ = O.quantize(W)
    xq, s_x, _, _ = O.quantize(X)
    dyq, s_dy, _, _ = O.quantize(dY)
    return dict(X=X, A=A, B=B, dY=dY, wq=wq, s_w=s_w, xq=xq, s_x=s_x, dyq=dyq, s_dy=s_dy)


def _run(c, precision, rnd=True):
    f = SP.separate_fwd(c["X"], c["A"], c["B"], c["xq"], c["s_x"], c["wq"], c["s_w"], precision, rnd=rnd)
    b = SP.separate_bwd(c["X"], c["dY"], c["A"], c["B"], f["S"], c["xq"], c["s_x"], c["dyq"], c["s_dy"], c["wq"],
                        c["s_w"], precision, rnd=rnd)
    return f, b


def test_matmul_f64_against_a_loop():
    rng = np.random.default_rng(0)
    a, b_nk, b_kn = rng.standard_normal((5, 7)), rng.standard_normal((3, 7)), rng.standard_normal((7, 3))
    loop = lambda a, bt: np.array([[sum(a[m, k] * bt[n][k] for k in range(a.shape[1])) for n in range(len(bt))]
                                   for m in range(a.shape[0])])
    np.testing.assert_allclose(O.matmul_f64(a, b_nk, True), loop(a, b_nk), rtol=1e-15, atol=0)
    np.testing.assert_allclose(O.matmul_f64(a, b_kn, False), loop(a, b_kn.T), rtol=1e-15, atol=0)


def test_unrounded_bf16_path_matches_autograd():
    torch = pytest.importorskip("torch")
    c = _case(1)
    f, b = _run(c, "bf16", rnd=False)
    X, A, B, dY = (torch.tensor(gen.bf16_bits_to_f32(c[k]).reshape(c[k].shape), dtype=torch.float64,
                                requires_grad=True) for k in ("X", "A", "B", "dY"))
    ylora = (X @ A.T) @ B.T  # the adapter layer kept beside the backbone
    (ylora * dY).sum().backward()
    np.testing.assert_allclose(f["Ylora"], ylora.detach().numpy(), rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(b["dXlora"], X.grad.numpy(), rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(b["dA"], A.grad.numpy(), rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(b["dB"], B.grad.numpy(), rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(f["Y"], f["Ybb"] + f["Ylora"], rtol=0, atol=0)


@pytest.mark.parametrize("precision", ["bf16", "fp8"])
def test_zero_adapters_reduce_to_the_backbone(precision):
    c = _case(2)
    c0 = dict(c, B=np.zeros_like(c["B"]))
    f, b = _run(c0, precision)
    assert np.array_equal(f["Y"], f["Ybb"]) and not f["Ylora"].any()
    assert np.array_equal(b["dX"], b["dXbb"]) and not b["G"].any() and not b["dA"].any()
    assert b["dB"].any()
    cA = dict(c, A=np.zeros_like(c["A"]))
    f, b = _run(cA, precision)
    assert not f["S"].any() and not f["Ylora"].any() and not b["dB"].any() and not b["dXlora"].any()
    assert np.array_equal(f["Y"], f["Ybb"]) and b["dA"].any()


def _grid(seed, shape, exp, planted_cols):
    """bf16 bits of values on the E4M3 grid times 2**exp, with 448 * 2**exp
    planted in the first `planted_cols` columns so that the tensor's scale
    is 2**-exp."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 0x7E, size=shape).astype(np.uint8) | (rng.integers(0, 2, size=shape) << 7).astype(np.uint8)
    v = DEC[codes] * 2.0 ** exp
    v[0, min(planted_cols, shape[1]) - 1] = 448.0 * 2.0 ** exp
    return _bf16(v)


def test_fp8_path_equals_bf16_path_when_every_quantization_is_lossless():
    M, N, K, r = 24, 32, 48, 16
    X = _grid(3, (M, K), -10, r)          # s_X = 2^10
    dY = _grid(4, (M, N), -14, r)         # s_dY = 2^14
    A = np.zeros((r, K), np.float32)
    A[np.arange(r), np.arange(r)] = 2.0 ** -3   # one-hot: S[m,i] = X[m,i] / 8, lossless at s_S = 2^13
    B = np.zeros((N, r), np.float32)
    B[np.arange(r), np.arange(r)] = 2.0 ** -2   # G[m,i] = dY[m,i] / 4, lossless at s_G = 2^16
    c = _case(5, M, N, K, r)
    c.update(X=X, dY=dY, A=_bf16(A), B=_bf16(B))
    c["xq"], c["s_x"], _, _ = O.quantize(X)
    c["dyq"], c["s_dy"], _, _ = O.quantize(dY)
    assert c["s_x"] == 2.0 ** 10 and c["s_dy"] == 2.0 ** 14
    f8, b8 = _run(c, "fp8")
    f16, b16 = _run(c, "bf16")
    assert f8["s_s"] == 2.0 ** 13 and b8["s_g"] == 2.0 ** 16
    for k in ("S", "Ylora", "Y"):
        assert np.array_equal(f8[k], f16[k]), k
    for k in ("G", "dXlora", "dX", "dB", "dA"):
        assert np.array_equal(b8[k], b16[k]), k
    assert f8["Ylora"].any() and b8["dB"].any() and b8["dA"].any()


def test_fp8_products_against_loops_over_decoded_codes():
    c = _case(6, M=6, N=8, K=16, r=4)
    f, b = _run(c, "fp8")
    sq, bq, s_s, s_b = f["sq"], f["bq"], float(f["s_s"]), float(f["s_b"])
    gq, aq, s_g, s_a = b["gq"], b["aq"], float(b["s_g"]), float(b["s_a"])
    dyq, xq, s_dy, s_x = c["dyq"], c["xq"], float(c["s_dy"]), float(c["s_x"])
    M, N, K, r = 6, 8, 16, 4
    r16 = lambda v: O.bf16_to_f64(O.bf16_round(np.array(v)))
    ylora = [[sum(DEC[sq[m, i]] * DEC[bq[n, i]] for i in range(r)) / (s_s * s_b) for n in range(N)] for m in range(M)]
    dxl = [[sum(DEC[gq[m, i]] * DEC[aq[i, k]] for i in range(r)) / (s_g * s_a) for k in range(K)] for m in range(M)]
    db = [[sum(DEC[dyq[m, n]] * DEC[sq[m, i]] for m in range(M)) / (s_dy * s_s) for i in range(r)] for n in range(N)]
    da = [[sum(DEC[gq[m, i]] * DEC[xq[m, k]] for m in range(M)) / (s_g * s_x) for k in range(K)] for i in range(r)]
    np.testing.assert_array_equal(f["Ylora"], r16(ylora))
    np.testing.assert_array_equal(b["dXlora"], r16(dxl))
    np.testing.assert_array_equal(b["dB"], r16(db))
    np.testing.assert_array_equal(b["dA"], r16(da))
    # S and G are the quantized products of the backbone's codes and the adapters' codes
    s = [[sum(DEC[xq[m, k]] * DEC[f["aq"][i, k]] for k in range(K)) / (s_x * float(f["s_a"])) for i in range(r)]
         for m in range(M)]
    np.testing.assert_array_equal(f["S"], r16(s))


def test_given_intermediates_are_used():
    c = _case(7)
    f = SP.separate_fwd(c["X"], c["A"], c["B"], c["xq"], c["s_x"], c["wq"], c["s_w"], "bf16")
    S2 = f["S"] * 2.0  # exact in bf16
    f2 = SP.separate_fwd(c["X"], c["A"], c["B"], c["xq"], c["s_x"], c["wq"], c["s_w"], "bf16", S_given=S2)
    np.testing.assert_array_equal(f2["Ylora"], f["Ylora"] * 2.0)
