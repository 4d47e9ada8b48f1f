"""Row-wise proxy update on the GPU against the oracle: bit-exact proxy,
codes, row mask and selected-row count."""

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


def _state(seed, N, K, r, p_std=1e-5, inc_std=1e-3):
    wq, s_w, _, _ = O.quantize(gen.normal_f32(seed, (N, K), 0.02))
    P = gen.normal_f32(seed + 1, (N, K), p_std) if p_std else np.zeros((N, K), np.float32)
    dB = gen.normal_bf16_bits(seed + 2, (N, r), inc_std)
    A = gen.normal_bf16_bits(seed + 3, (r, K), 0.01)
    return wq, s_w, P, dB, A


def _gpu(wq, s_w, P, dB, A, flags=F.PROXY_ACCUMULATE | F.PROXY_SELECT):
    w = dev_u8(wq)
    p = dev_f32(P)
    st = status_word()
    mask, cnt = F.falqon_proxy_update(w, dev_f32([s_w]), p, dev_bf16(dB), dev_bf16(A), flags=flags,
                                      dev_status=st)
    torch.cuda.synchronize()
    return (host(w), host(p), None if mask is None else host(mask),
            None if cnt is None else int(host(cnt)[0]), int(host(st)[0]))


def _compare(gpu, ref):
    w, p, mask, cnt, st = gpu
    rw, rp, rmask, rcnt = ref
    np.testing.assert_array_equal(p.view(np.uint32), rp.view(np.uint32))
    np.testing.assert_array_equal(w, rw)
    if rmask is not None:
        np.testing.assert_array_equal(mask, rmask)
        assert cnt == rcnt
    assert st == 0


@pytest.mark.parametrize("N,K,r", [
    (512, 512, 16),     # one 256-column block per row group
    (37, 48, 5),        # tiny, ragged rows
    (64, 272, 33),      # odd r; K ends in a partial 256-column block
    (130, 512, 64),
    (96, 1024, 100),    # r beyond one 64-wide staging chunk
    (70, 2048, 64),     # rows not a multiple of the 32-row group
    (40, 11008, 16),    # the down projection's K (43 column blocks)
    (64, 512, 1100),    # large rank: many staging chunks
    (160, 32768, 64),   # persistent CTAs whose tiles span column blocks
    (20, 65536, 8),     # one row group: every tile starts a new column block
])
def test_accumulate_and_select(cuda_device, N, K, r):
    O.set_threads(os.cpu_count() or 8)
    case = _state(N + K + r, N, K, r)
    ref = O.proxy_update(*case)
    _compare(_gpu(*case), ref)
    assert 0 < ref[3] <= N


def test_selection_partial_and_none(cuda_device):
    # small increments: some rows selected, not all; zero increment: none
    case = _state(3, 256, 256, 16, p_std=1e-6, inc_std=1e-4)
    ref = O.proxy_update(*case)
    assert 0 < ref[3] < 256
    _compare(_gpu(*case), ref)
    wq, s_w, P, dB, A = case
    zero = (wq, s_w, np.zeros_like(P), np.zeros_like(dB), A)
    ref0 = O.proxy_update(*zero)
    assert ref0[3] == 0
    _compare(_gpu(*zero), ref0)


def test_accumulate_only_and_select_only(cuda_device):
    wq, s_w, P, dB, A = _state(4, 128, 256, 16)
    g = _gpu(wq, s_w, P, dB, A, flags=F.PROXY_ACCUMULATE)
    Pn = O.proxy_accumulate(P, dB, A)
    np.testing.assert_array_equal(g[1].view(np.uint32), Pn.view(np.uint32))
    np.testing.assert_array_equal(g[0], wq)
    g2 = _gpu(wq, s_w, Pn, dB, A, flags=F.PROXY_SELECT)
    _compare(g2, O.proxy_select(wq, s_w, Pn))


def test_planted_single_update(cuda_device):
    wq, s_w, _, dB, A = _state(5, 64, 128, 8)
    P = np.zeros_like(wq, dtype=np.float32)
    n, k = 17, 45
    c = 0x30
    wq[n, k] = c
    P[n, k] = np.float32((DEC[c + 1] - DEC[c]) / np.float64(s_w))
    g = _gpu(wq, s_w, P, dB, A, flags=F.PROXY_SELECT)
    ref = O.proxy_select(wq, s_w, P)
    assert ref[3] == 1 and ref[0][n, k] == c + 1
    _compare(g, ref)


def test_full_size_attention_projection(cuda_device):
    O.set_threads(os.cpu_count() or 8)
    case = _state(6, 4096, 4096, 64, p_std=1e-5, inc_std=1e-4)
    _compare(_gpu(*case), O.proxy_update(*case))


def test_twenty_step_trajectory_matches(cuda_device):
    """Both sides run 20 steps from the same state with the same per-step
    increments (seeded, independent of either side)."""
    N, K, r = 192, 384, 16
    wq, s_w, P, _, A = _state(7, N, K, r, p_std=0)
    w, p = dev_u8(wq), dev_f32(P)
    s_dev, A_dev = dev_f32([s_w]), dev_bf16(A)
    for step in range(20):
        dB = gen.normal_bf16_bits(1000 + step, (N, r), 3e-4)
        mask, cnt = F.falqon_proxy_update(w, s_dev, p, dev_bf16(dB), A_dev)
        wq, P, rmask, rcnt = O.proxy_update(wq, s_w, P, dB, A)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host(w), wq)
        np.testing.assert_array_equal(host(p).view(np.uint32), P.view(np.uint32))
        np.testing.assert_array_equal(host(mask), rmask)
        assert int(host(cnt)[0]) == rcnt


@pytest.mark.parametrize("N,K,r", [
    (256, 256, 16),     # persistent kernel
    (37, 48, 5),        # grid kernel, ragged
    (70, 2048, 64),
    (96, 1024, 100),
])
def test_keep_residual_matches_oracle(cuda_device, N, K, r):
    """Error-feedback clear (C-14): codes as the clearing rule, the proxy keeps
    what the new codes did not apply."""
    O.set_threads(os.cpu_count() or 8)
    case = _state(N + K + r + 7, N, K, r, p_std=1e-6, inc_std=1e-4)
    ref = O.proxy_update(*case, keep_residual=True)
    assert 0 < ref[3] <= N
    flags = F.PROXY_ACCUMULATE | F.PROXY_SELECT | F.PROXY_KEEP_RESIDUAL
    _compare(_gpu(*case, flags=flags), ref)


def test_keep_residual_trajectory_matches(cuda_device):
    N, K, r = 128, 512, 16
    wq, s_w, P, _, A = _state(17, N, K, r, p_std=0)
    w, p = dev_u8(wq), dev_f32(P)
    s_dev, A_dev = dev_f32([s_w]), dev_bf16(A)
    flags = F.PROXY_ACCUMULATE | F.PROXY_SELECT | F.PROXY_KEEP_RESIDUAL
    for step in range(10):
        dB = gen.normal_bf16_bits(3000 + step, (N, r), 3e-4)
        mask, cnt = F.falqon_proxy_update(w, s_dev, p, dev_bf16(dB), A_dev, flags=flags)
        wq, P, rmask, rcnt = O.proxy_update(wq, s_w, P, dB, A, keep_residual=True)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host(w), wq)
        np.testing.assert_array_equal(host(p).view(np.uint32), P.view(np.uint32))
        np.testing.assert_array_equal(host(mask), rmask)
        assert int(host(cnt)[0]) == rcnt


@pytest.mark.parametrize("N,K,r,steps,inc", [
    (192, 384, 16, 12, 3e-4),    # persistent kernel, nearly every row selected every step
    (192, 384, 16, 12, 3e-5),    # about a third selected: rows leave the mask at most steps
    (37, 48, 5, 8, 3e-3),        # grid kernel (r % 8 != 0), ragged
    (96, 1024, 100, 6, 1e-3),    # grid kernel, r above one staging chunk
    (130, 512, 64, 10, 3e-6),    # about a tenth selected
])
def test_deferred_clear_trajectory_matches(cuda_device, N, K, r, steps, inc):
    """DEFER_CLEAR carries the clear of the selected rows to the next call
    through row_mask.  Every step: codes, row mask and count bit-identical to
    the oracle's eager update, and the proxy the caller holds (P with the
    rows marked in row_mask read as +0) bit-identical to the oracle's P."""
    O.set_threads(os.cpu_count() or 8)
    wq, s_w, P, _, A = _state(N + K + r + 31, N, K, r, p_std=0)
    w, p = dev_u8(wq), dev_f32(P)
    s_dev, A_dev = dev_f32([s_w]), dev_bf16(A)
    mask = torch.zeros(N, dtype=torch.uint8, device="cuda:0")  # no earlier selection
    st = status_word()
    flags = F.PROXY_ACCUMULATE | F.PROXY_SELECT | F.PROXY_DEFER_CLEAR
    seen = 0
    for step in range(steps):
        dB = gen.normal_bf16_bits(5000 + 17 * N + step, (N, r), inc)
        _, cnt = F.falqon_proxy_update(w, s_dev, p, dev_bf16(dB), A_dev, flags=flags, row_mask=mask,
                                       dev_status=st)
        wq, P, rmask, rcnt = O.proxy_update(wq, s_w, P, dB, A)
        torch.cuda.synchronize()
        hm = host(mask)
        held = host(p).copy()
        held[hm != 0] = 0.0  # the deferred clear: +0
        np.testing.assert_array_equal(host(w), wq)
        np.testing.assert_array_equal(hm, rmask)
        assert int(host(cnt)[0]) == rcnt
        np.testing.assert_array_equal(held.view(np.uint32), P.view(np.uint32))
        seen += rcnt
    assert int(host(st)[0]) == 0
    assert seen > 0
