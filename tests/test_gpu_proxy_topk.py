"""Proxy update with top-k row selection on the GPU against the oracle
(C-13): bit-exact proxy, codes, row mask and selected-row count."""

import os

import numpy as np
import pytest
import torch

import fp8_quantized_lora_b200 as F
import oracle as O
from gpu_util import dev_bf16, dev_f32, dev_u8, host, status_word
from synthetic import gen

pytestmark = pytest.mark.gpu

DEC = np.array([O.e4m3_decode(c) for c in range(256)])


def _state(seed, N, K, r, p_std=1e-6, inc_std=1e-4):
    wq, s_w, _, _ = O.quantize(gen.normal_f32(seed, (N, K), 0.02))
    P = gen.normal_f32(seed + 1, (N, K), p_std) if p_std else np.zeros((N, K), np.float32)
    dB = gen.normal_bf16_bits(seed + 2, (N, r), inc_std)
    A = gen.normal_bf16_bits(seed + 3, (r, K), 0.01)
    return wq, s_w, P, dB, A


def _gpu(wq, s_w, P, dB, A, k):
    w = dev_u8(wq)
    p = dev_f32(P)
    st = status_word()
    mask, cnt = F.falqon_proxy_update_topk(w, dev_f32([s_w]), p, dev_bf16(dB), dev_bf16(A), k, dev_status=st)
    torch.cuda.synchronize()
    return host(w), host(p), host(mask), int(host(cnt)[0]), int(host(st)[0])


def _compare(gpu, ref):
    w, p, mask, cnt, st = gpu
    rw, rp, rmask, rcnt = ref
    np.testing.assert_array_equal(mask, rmask)
    assert cnt == rcnt
    np.testing.assert_array_equal(p.view(np.uint32), rp.view(np.uint32))
    np.testing.assert_array_equal(w, rw)
    assert st == 0


@pytest.mark.parametrize("N,K,r,k", [
    (256, 256, 16, 32),     # persistent kernel, some candidates left out
    (37, 48, 5, 4),         # tiny and ragged; odd r: the grid kernel
    (130, 512, 64, 1),
    (70, 2048, 64, 17),     # rows not a multiple of the 32-row group
    (96, 1024, 100, 50),    # r beyond one staging chunk (grid kernel)
    (40, 11008, 16, 8),     # many column blocks per row
    (1500, 256, 8, 600),    # several passes of the selection walk
    (200, 512, 16, 0),      # k = 0: accumulate only
    (200, 512, 16, 10000),  # k beyond N: every candidate (the threshold rule)
])
def test_topk_matches_oracle(cuda_device, N, K, r, k):
    O.set_threads(os.cpu_count() or 8)
    case = _state(N + K + r + k, N, K, r)
    ref = O.proxy_update_topk(*case, k)
    if 0 < k < N:
        assert 0 < ref[3] <= k
    _compare(_gpu(*case, k), ref)


def test_topk_ties_go_to_the_lower_index(cuda_device):
    """Planted scores with ties: rows 3, 40 and 77 change 5 codes each, row 9
    changes 7, row 50 changes 2; k = 3 takes rows 9, 3 and 40."""
    N, K, r = 96, 256, 8
    wq = np.full((N, K), 0x30, dtype=np.uint8)
    P = np.zeros((N, K), dtype=np.float32)
    s_w = np.float32(1.0)
    step = np.float32(DEC[0x31] - DEC[0x30])
    for n, s in ((3, 5), (40, 5), (77, 5), (9, 7), (50, 2)):
        P[n, 100:100 + s] = step
    dB = np.zeros((N, r), dtype=np.uint16)
    A = gen.normal_bf16_bits(5, (r, K), 0.01)
    ref = O.proxy_update_topk(wq, s_w, P, dB, A, 3)
    assert np.flatnonzero(ref[2]).tolist() == [3, 9, 40]
    _compare(_gpu(wq, s_w, P, dB, A, 3), ref)


def test_topk_full_size_attention_projection(cuda_device):
    O.set_threads(os.cpu_count() or 8)
    case = _state(8, 4096, 4096, 64, p_std=1e-7, inc_std=2e-5)
    ref = O.proxy_update_topk(*case, 256)
    assert ref[3] == 256
    _compare(_gpu(*case, 256), ref)


def test_topk_trajectory_matches(cuda_device):
    """Twelve steps from the same state with the same seeded increments."""
    N, K, r, k = 160, 512, 16, 24
    wq, s_w, P, _, A = _state(9, N, K, r, p_std=0)
    w, p = dev_u8(wq), dev_f32(P)
    s_dev, A_dev = dev_f32([s_w]), dev_bf16(A)
    for step in range(12):
        dB = gen.normal_bf16_bits(2000 + step, (N, r), 1e-4)
        mask, cnt = F.falqon_proxy_update_topk(w, s_dev, p, dev_bf16(dB), A_dev, k)
        wq, P, rmask, rcnt = O.proxy_update_topk(wq, s_w, P, dB, A, k)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host(mask), rmask)
        assert int(host(cnt)[0]) == rcnt
        np.testing.assert_array_equal(host(w), wq)
        np.testing.assert_array_equal(host(p).view(np.uint32), P.view(np.uint32))


@pytest.mark.parametrize("N,K,r,k", [
    (256, 256, 16, 32),
    (37, 48, 5, 4),
    (70, 2048, 64, 17),
])
def test_topk_keep_residual_matches_oracle(cuda_device, N, K, r, k):
    O.set_threads(os.cpu_count() or 8)
    case = _state(N + K + r + k + 3, N, K, r)
    ref = O.proxy_update_topk(*case, k, keep_residual=True)
    w = dev_u8(case[0])
    p = dev_f32(case[2])
    st = status_word()
    mask, cnt = F.falqon_proxy_update_topk(w, dev_f32([case[1]]), p, dev_bf16(case[3]), dev_bf16(case[4]), k,
                                           keep_residual=True, dev_status=st)
    torch.cuda.synchronize()
    _compare((host(w), host(p), host(mask), int(host(cnt)[0]), int(host(st)[0])), ref)
