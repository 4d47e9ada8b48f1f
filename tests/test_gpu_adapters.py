"""Adapter gradients dB and dA against the oracle, within the float acceptance
rule: the rank-on-M kernel (tcgen05 kind::f16 with in-smem E4M3 expansion)
and, from r = 512, the bf16-GEMM path (codes expanded once)."""

import os

import numpy as np
import pytest
import torch

import fp8_quantized_lora_b200 as F
import oracle as O
from gpu_util import dev_bf16, dev_f32, dev_u8, host_bf16_bits, status_word
from synthetic import WORKLOADS, gen, layer_inputs

pytestmark = pytest.mark.gpu


def _case(seed, M, N, K, r, b_std=1e-3):
    xq, s_x, _, _ = O.quantize(gen.normal_bf16_bits(seed, (M, K), 1.0))
    dyq, s_dy, _, _ = O.quantize(gen.normal_bf16_bits(seed + 1, (M, N), 1e-3))
    A = gen.normal_bf16_bits(seed + 2, (r, K), 0.01)
    B = gen.normal_bf16_bits(seed + 3, (N, r), b_std) if b_std else np.zeros((N, r), np.uint16)
    return xq, s_x, dyq, s_dy, A, B


def _gpu(xq, s_x, dyq, s_dy, A, B, want_da=True):
    st = status_word()
    _, dA, dB = F.falqon_linear_bwd(dev_u8(dyq), dev_f32([s_dy]), None, None, dev_u8(xq),
                                    dev_f32([s_x]), dev_bf16(A), dev_bf16(B), dx=None,
                                    dA=True if want_da else None, dB=True, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return (host_bf16_bits(dA) if want_da else None), host_bf16_bits(dB)


def _oracle(xq, s_x, dyq, s_dy, A, B):
    t64, _ = O.adapter_t(xq, s_x, A)
    db = O.adapter_db(dyq, s_dy, t64=t64)
    u64, _ = O.adapter_u(dyq, s_dy, B)
    da = O.adapter_da(xq, s_x, u64=u64)
    return da, db


CASES = [
    (256, 512, 512, 16),    # the tiny parity workload's shapes
    (200, 272, 336, 32),    # ragged M, N, K; r below the 64-wide tile
    (130, 128, 192, 64),
    (512, 256, 384, 80),    # r not a power of two (128-wide tile, 48 padded columns)
    (256, 384, 256, 256),
    (128, 256, 512, 320),   # two r tiles
    (2048, 256, 4096, 16),  # 16 row tiles: split-K clusters of 8
    (1000, 4096, 1024, 64), # many dB/dA^T tiles, few splits
    (3, 256, 512, 16),      # fewer tokens than one K block of dB / dA
    (333, 512, 768, 192),   # odd M (padded T/U rows); r over one rank tile
    # from r = 512 (M a multiple of 8) the products run on the bf16 GEMM: codes
    # expanded once, T and U in float32, hi + lo planes stacked in dB / dA
    (520, 512, 768, 512),
    (1024, 272, 1024, 576),  # N not a multiple of the 256-wide tile
    (8, 256, 256, 512),      # one token tile
    (333, 256, 512, 512),    # M not a multiple of 8: the rank-on-M kernel at a large rank
]


@pytest.mark.parametrize("M,N,K,r", CASES)
def test_db_and_da(cuda_device, M, N, K, r):
    O.set_threads(os.cpu_count() or 8)
    case = _case(M + N + r, M, N, K, r)
    da, db = _gpu(*case)
    rda, rdb = _oracle(*case)
    rep_b = O.tolerance_report(db, rdb)
    rep_a = O.tolerance_report(da, rda)
    assert rep_b["ok"], ("dB", rep_b)
    assert rep_a["ok"], ("dA", rep_a)


def test_zero_b_gives_exactly_zero_da(cuda_device):
    case = _case(5, 256, 512, 512, 16, b_std=0)
    da, db = _gpu(*case)
    assert np.all((da & 0x7FFF) == 0)
    _, rdb = _oracle(*case)
    assert O.tolerance_report(db, rdb)["ok"]


def test_db_only_skips_da(cuda_device):
    case = _case(6, 128, 256, 256, 16)
    da, db = _gpu(*case, want_da=False)
    assert da is None
    _, rdb = _oracle(*case)
    assert O.tolerance_report(db, rdb)["ok"]


@pytest.mark.parametrize("name", ["llama7b_attn_proj_4096x4096x4096_r64"])
def test_llama_attention_full_size(cuda_device, name):
    """The bench's workload at full size: the oracle computes all of dB and dA."""
    O.set_threads(os.cpu_count() or 8)
    wl = WORKLOADS[name]
    d = layer_inputs(wl, wl.layers[0], with_b=True)
    xq, s_x, _, _ = O.quantize(d["X"])
    dyq, s_dy, _, _ = O.quantize(d["dY"])
    case = (xq, s_x, dyq, s_dy, d["A"], d["B"])
    da, db = _gpu(*case)
    rda, rdb = _oracle(*case)
    assert O.tolerance_report(db, rdb)["ok"]
    assert O.tolerance_report(da, rda)["ok"]


def _every_code(shape, offset):
    """Codes cycling through all 254 non-NaN E4M3 codes."""
    valid = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    idx = (np.arange(shape[0] * shape[1]) * 7 + offset) % valid.size
    return valid[idx].reshape(shape)


@pytest.mark.parametrize("r", [32, 512])
def test_every_code_expands_exactly(cuda_device, r):
    """Each operand holds every non-NaN code (subnormals, zeros of both signs,
    +-448), so each code's expansion to bf16 enters both products (both
    paths: the in-tile expansion and, at r = 512, the expansion pass)."""
    M, N, K = 256, 384, 512
    xq, dyq = _every_code((M, K), 0), _every_code((M, N), 3)
    s_x, s_dy = np.float32(3.0), np.float32(0.5)
    A = gen.normal_bf16_bits(11, (r, K), 0.01)
    B = gen.normal_bf16_bits(12, (N, r), 0.01)
    case = (xq, s_x, dyq, s_dy, A, B)
    da, db = _gpu(*case)
    rda, rdb = _oracle(*case)
    assert O.tolerance_report(db, rdb)["ok"]
    assert O.tolerance_report(da, rda)["ok"]


@pytest.mark.parametrize("r", [16, 512])
def test_nan_code_propagates(cuda_device, r):
    """A NaN code in Xq poisons its row of T (hence all of dB) and its column
    of dA, on both sides; everything else still matches."""
    M, N, K = 128, 256, 256
    xq, s_x, dyq, s_dy, A, B = _case(13, M, N, K, r)
    xq = xq.copy()
    xq[5, 77] = 0xFF
    da, db = _gpu(xq, s_x, dyq, s_dy, A, B)
    rda, rdb = _oracle(xq, s_x, dyq, s_dy, A, B)

    def isnan(bits):
        return ((bits & 0x7F80) == 0x7F80) & ((bits & 0x007F) != 0)

    assert np.array_equal(isnan(db), np.isnan(rdb)) and np.isnan(rdb).all()
    assert np.array_equal(isnan(da), np.isnan(rda))
    assert np.isnan(rda[:, 77]).all() and not np.isnan(np.delete(rda, 77, axis=1)).any()
    assert O.tolerance_report(np.delete(da, 77, axis=1), np.delete(rda, 77, axis=1))["ok"]
