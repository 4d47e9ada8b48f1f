"""Forward and dX GEMMs (tcgen05 kind::f8f6f4) against the oracle, within the
float acceptance rule of oracle/tolerance.py."""

import os

import numpy as np
import pytest
import torch

import fp8_quantized_lora_b200 as F
import oracle as O
from gpu_util import dev_f32, dev_u8, host_bf16_bits, sample_rows, status_word
from synthetic import gen

pytestmark = pytest.mark.gpu


def _codes(seed, shape, std=1.0):
    x = gen.normal_bf16_bits(seed, shape, std)
    c, s, _, _ = O.quantize(x)
    return c, s


def _fwd(xq, s_x, wq, s_w):
    st = status_word()
    y = F.falqon_linear_fwd(dev_u8(xq), dev_f32([s_x]), dev_u8(wq), dev_f32([s_w]), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return host_bf16_bits(y)


def _dx(dyq, s_dy, wq, s_w):
    st = status_word()
    dx, _, _ = F.falqon_linear_bwd(dev_u8(dyq), dev_f32([s_dy]), dev_u8(wq), dev_f32([s_w]),
                                   None, None, None, None, dx=True, dA=None, dB=None, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return host_bf16_bits(dx)


def _assert_close(G, R, what):
    rep = O.tolerance_report(G, R)
    assert rep["ok"], (what, rep)


SHAPES = [
    (256, 512, 512),     # the tiny parity workload
    (200, 272, 336),     # ragged in every dimension: M, N and K tails
    (1, 16, 16),         # smallest legal problem
    (130, 256, 128),     # one row past a tile
    (384, 528, 2048),    # long K, N one block past two tiles
]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_forward(cuda_device, M, N, K):
    xq, s_x = _codes(100 + M, (M, K))
    wq, s_w = _codes(200 + N, (N, K), 0.02)
    _assert_close(_fwd(xq, s_x, wq, s_w), O.linear_fwd(xq, s_x, wq, s_w), (M, N, K))


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_dx(cuda_device, M, N, K):
    dyq, s_dy = _codes(300 + M, (M, N), 1e-3)
    wq, s_w = _codes(400 + N, (N, K), 0.02)
    _assert_close(_dx(dyq, s_dy, wq, s_w), O.linear_dx(dyq, s_dy, wq, s_w), (M, N, K))


def test_partial_last_wave_runs_as_half_tiles(cuda_device):
    """A grid whose last wave is partial: 19 x 5 = 95 output tiles of
    256 x 256 on the SM pairs (74 on a 148-SM B200), the last M band half
    empty.  In the forward the 21 tiles of the last wave run as 42 halves
    (256 x 128: N = 128 pair MMAs, 64 B rows per CTA); dX (MN-major B) runs
    them whole.  Every output element is compared, the forward and dX both."""
    O.set_threads(os.cpu_count() or 8)
    M, N, K = 37 * 128, 5 * 256, 256
    xq, s_x = _codes(811, (M, K))
    wq, s_w = _codes(812, (N, K), 0.02)
    _assert_close(_fwd(xq, s_x, wq, s_w), O.linear_fwd(xq, s_x, wq, s_w), "fwd")
    dyq, s_dy = _codes(813, (M, K), 1e-3)  # dX [M, N]: contraction over K here
    wq2, s_w2 = _codes(814, (K, N), 0.02)
    _assert_close(_dx(dyq, s_dy, wq2, s_w2), O.linear_dx(dyq, s_dy, wq2, s_w2), "dx")


def test_forward_identity_backbone_is_exact(cuda_device):
    M, K = 130, 256
    xq, s_x = _codes(7, (M, K))
    wq = np.zeros((K, K), dtype=np.uint8)
    np.fill_diagonal(wq, 0x38)
    y = _fwd(xq, s_x, wq, np.float32(1.0))
    np.testing.assert_array_equal(y, O.bf16_round(O.linear_fwd(xq, s_x, wq, np.float32(1.0))))


@pytest.mark.parametrize("M,N,K", [(4096, 4096, 4096), (8192, 11008, 4096), (8192, 4096, 11008)])
def test_llama_shapes_sampled_rows(cuda_device, M, N, K):
    """Full Llama-7B shapes in the bench's launch configuration; the oracle
    computes a row sample that touches every M tile and the last row."""
    O.set_threads(os.cpu_count() or 8)
    xq, s_x = _codes(500 + N, (M, K))
    wq, s_w = _codes(600 + K, (N, K), 0.02)
    y = _fwd(xq, s_x, wq, s_w)
    rows = sample_rows(M, 512)
    for r0 in rows:
        _assert_close(y[r0], O.linear_fwd(xq, s_x, wq, s_w, rows=(r0, r0 + 1))[0], ("fwd", r0))
    dyq, s_dy = _codes(700 + N, (M, N), 1e-3)
    dx = _dx(dyq, s_dy, wq, s_w)
    for r0 in rows:
        _assert_close(dx[r0], O.linear_dx(dyq, s_dy, wq, s_w, rows=(r0, r0 + 1))[0], ("dx", r0))


@pytest.mark.parametrize("M,N,K", [
    (2048, 3328, 256),   # 8 x 13 = 104 tiles of 256 x 256: 74 whole, 30 tiles as 60 halves
    (512, 4096, 384),    # 2 x 16 = 32 tiles: fewer tiles than pairs, K not a multiple of 256
    (300, 208, 144),     # one tile, both operands ragged: rows and columns past the ends
])
def test_pair_tiles_and_tails(cuda_device, M, N, K):
    """The SM-pair GEMM (256 x 256 tiles, each CTA staging 128 rows of A and
    128 columns of B) on grids with a partial last wave, fewer tiles than
    pairs, and tiles that overhang both operands."""
    O.set_threads(os.cpu_count() or 8)
    xq, s_x = _codes(900 + M, (M, K))
    wq, s_w = _codes(901 + N, (N, K), 0.02)
    _assert_close(_fwd(xq, s_x, wq, s_w), O.linear_fwd(xq, s_x, wq, s_w), ("fwd", M, N, K))
    dyq, s_dy = _codes(902 + M, (M, K), 1e-3)  # dX [M, N]: contraction over K here
    wq2, s_w2 = _codes(903 + N, (K, N), 0.02)
    _assert_close(_dx(dyq, s_dy, wq2, s_w2), O.linear_dx(dyq, s_dy, wq2, s_w2), ("dx", M, N, K))
