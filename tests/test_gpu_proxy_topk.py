"""Top-k proxy update over the r rank components on the GPU against the
oracle (C-13): bit-exact proxy rows, codes, component mask, merged count and
status word."""

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
ACC, SEL = F.PROXY_ACCUMULATE, F.PROXY_SELECT


def _case(seed, N, K, r, q_std=0.05, inc_std=0.01):
    """Codes of W ~ N(0, 0.02), a proxy Q [r, N] ~ N(0, q_std), an increment
    dB_inc [N, r] ~ N(0, inc_std) (bf16) and A ~ N(0, 0.01) (bf16): large
    enough for a merge of a few components to move codes."""
    wq, s_w, _, _ = O.quantize(gen.normal_f32(seed, (N, K), 0.02))
    Q = gen.normal_f32(seed + 1, (r, N), q_std)
    dB = gen.normal_bf16_bits(seed + 2, (N, r), inc_std)
    A = gen.normal_bf16_bits(seed + 3, (r, K), 0.01)
    return wq, s_w, Q, dB, A


def _gpu(wq, s_w, Q, dB, A, k, flags=ACC | SEL):
    w, q, st = dev_u8(wq), dev_f32(Q), status_word()
    mask, cnt = F.falqon_proxy_update_topk(w, dev_f32([s_w]), q, dev_bf16(dB), dev_bf16(A), k, flags=flags,
                                           dev_status=st)
    torch.cuda.synchronize()
    return (host(w), host(q), None if mask is None else host(mask), None if cnt is None else int(host(cnt)[0]),
            int(host(st)[0]))


def _compare(gpu, ref, select=True):
    w, q, mask, cnt, st = gpu
    rw, rq, rmask, rcnt, rst = ref
    np.testing.assert_array_equal(q.view(np.uint32), rq.view(np.uint32))
    np.testing.assert_array_equal(w, rw)
    if select:
        np.testing.assert_array_equal(mask, rmask)
        assert cnt == rcnt
    assert st == rst


@pytest.mark.parametrize("N,K,r,k", [
    (256, 256, 16, 4),      # one column block
    (37, 48, 5, 2),         # ragged N (not a multiple of 32 or 64), odd r, K below a block
    (130, 512, 64, 16),     # the bench's r, k = r/4
    (70, 2048, 64, 17),
    (96, 1024, 100, 50),    # r beyond one 32-component accumulation block
    (64, 512, 200, 130),    # more than one 64-component merge chunk
    (40, 11008, 16, 8),     # many column blocks, K not a multiple of 256
    (1500, 256, 8, 3),      # many row groups
    (200, 512, 16, 0),      # k = 0: accumulate, choose nothing
    (200, 512, 16, 10000),  # k beyond r: every component with a positive score
])
def test_topk_matches_oracle(cuda_device, N, K, r, k):
    O.set_threads(os.cpu_count() or 8)
    case = _case(N + K + r + k, N, K, r)
    ref = O.proxy_update_topk(*case, k)
    if k > 0:
        assert ref[3] == min(k, r)
        assert (ref[0] != case[0]).any(), "the merge should move some codes"
    _compare(_gpu(*case, k), ref)


@pytest.mark.parametrize("flags", [ACC, SEL])
def test_topk_single_steps(cuda_device, flags):
    """ACCUMULATE alone (a float32 add, no choice) and SELECT alone (no add)."""
    case = _case(5, 96, 512, 24)
    ref = O.proxy_update_topk(*case, 6, accumulate=bool(flags & ACC), select=bool(flags & SEL))
    _compare(_gpu(*case, 6, flags=flags), ref, select=bool(flags & SEL))


def test_topk_ties_go_to_the_lower_index(cuda_device):
    """Components 3, 9 and 12 carry the same score (the same Q row scaled by
    -1 or moved, A rows equal up to sign); 5 carries a larger one; k = 3 takes
    5, 3 and 9."""
    N, K, r = 64, 256, 16
    wq, s_w, Q, dB, A = _case(6, N, K, r, q_std=1e-3)
    base_q = gen.normal_f32(60, (N,), 0.05)
    base_a = gen.normal_bf16_bits(61, (K,), 0.01)
    for i, sgn in ((3, 1), (9, -1), (12, 1)):
        Q[i] = sgn * np.roll(base_q, i)
        A[i] = base_a ^ np.uint16(0x8000 if sgn < 0 else 0)
    Q[5] = 2 * base_q
    A[5] = base_a
    ref = O.proxy_update_topk(wq, s_w, Q, dB, A, 3, accumulate=False)
    assert np.flatnonzero(ref[2]).tolist() == [3, 5, 9]
    _compare(_gpu(wq, s_w, Q, dB, A, 3, flags=SEL), ref)


def test_topk_full_size_attention_projection(cuda_device):
    """The bench's shape: N = K = 4096, r = 64, k = 16, compared in full."""
    O.set_threads(os.cpu_count() or 8)
    case = _case(8, 4096, 4096, 64)
    ref = O.proxy_update_topk(*case, 16)
    assert ref[3] == 16
    _compare(_gpu(*case, 16), ref)


def test_topk_large_rank(cuda_device):
    """r = 8192 (the rank sweep's largest): the choice runs over 8192 scores
    and the merge over several chunks of components."""
    O.set_threads(os.cpu_count() or 8)
    case = _case(9, 48, 64, 8192, q_std=0.01)
    ref = O.proxy_update_topk(*case, 150)
    assert ref[3] == 150
    _compare(_gpu(*case, 150), ref)


def test_topk_trajectory_matches(cuda_device):
    """Twelve steps from the same state with the same seeded increments."""
    N, K, r, k = 160, 512, 16, 4
    wq, s_w, Q, _, A = _case(10, N, K, r)
    Q = np.zeros_like(Q)
    w, q = dev_u8(wq), dev_f32(Q)
    s_dev, A_dev = dev_f32([s_w]), dev_bf16(A)
    for step in range(12):
        dB = gen.normal_bf16_bits(2000 + step, (N, r), 0.02)
        mask, cnt = F.falqon_proxy_update_topk(w, s_dev, q, dev_bf16(dB), A_dev, k)
        wq, Q, rmask, rcnt, _ = O.proxy_update_topk(wq, s_w, Q, dB, A, k)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host(mask), rmask)
        assert int(host(cnt)[0]) == rcnt
        np.testing.assert_array_equal(host(w), wq)
        np.testing.assert_array_equal(host(q).view(np.uint32), Q.view(np.uint32))


def test_topk_nonfinite_proxy_sets_status(cuda_device):
    case = list(_case(11, 64, 256, 16))
    case[2] = case[2].copy()
    case[2][7, 3] = np.inf
    ref = O.proxy_update_topk(*case, 2, accumulate=False)
    assert ref[4] == O.STATUS_NONFINITE and ref[2][7] == 1
    _compare(_gpu(*case, 2, flags=SEL), ref)
