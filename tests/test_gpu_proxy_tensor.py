"""Proxy accumulation on the tensor cores (FALQON_PROXY_TENSOR), the large-r
form of C-9: P = fl32(P + dB_inc . A) with bf16 products summed in float32
in the hardware's order.  No fixed summation order reproduces that order,
so P is checked against the exact (float64) P + dB_inc . A within the
float32 bound of an r-term sum,

    |P_gpu - (P + D)| <= r 2^-23 sum_i |b_i a_i| + 2^-23 |P + D|,

and the selection (C-10, C-11) is then checked bit-exact given the GPU's P."""

import os

import numpy as np
import pytest
import torch

import fp8_quantized_lora_b200 as F
import oracle as O
from gpu_util import dev_bf16, dev_f32, dev_u8, host, status_word
from synthetic import gen

pytestmark = pytest.mark.gpu


def _case(seed, N, K, r, p_std=1e-4, inc_std=2e-3):
    wq, s_w, _, _ = O.quantize(gen.normal_f32(seed, (N, K), 0.02))
    P = gen.normal_f32(seed + 1, (N, K), p_std)
    dB = gen.normal_bf16_bits(seed + 2, (N, r), inc_std)
    A = gen.normal_bf16_bits(seed + 3, (r, K), 0.01)
    return wq, s_w, P, dB, A


@pytest.mark.parametrize("N,K,r", [
    (256, 512, 256),
    (200, 272, 512),     # ragged rows and columns
    (512, 1024, 1024),
    (128, 256, 8192),    # the rank sweep's largest rank
    (96, 512, 24),       # a small r that is a multiple of 8 only
])
def test_tensor_accumulation_within_bound_then_exact_selection(cuda_device, N, K, r):
    O.set_threads(os.cpu_count() or 8)
    wq, s_w, P, dB, A = _case(N + K + r, N, K, r)
    w, p, st = dev_u8(wq), dev_f32(P), status_word()
    F.falqon_proxy_update(w, dev_f32([s_w]), p, dev_bf16(dB), dev_bf16(A),
                          flags=F.PROXY_ACCUMULATE | F.PROXY_TENSOR, dev_status=st)
    torch.cuda.synchronize()
    Pg = host(p)
    Bf = O.bf16_to_f64(dB)
    Af = O.bf16_to_f64(A)
    D = O.matmul_f64(Bf, Af, False)
    absD = O.matmul_f64(np.abs(Bf), np.abs(Af), False)
    exact = P.astype(np.float64) + D
    bound = r * 2.0 ** -23 * absD + 2.0 ** -23 * np.abs(exact)
    err = np.abs(Pg.astype(np.float64) - exact)
    assert np.all(err <= bound), float(np.max(err / np.maximum(bound, 1e-300)))
    assert np.array_equal(host(w), wq)  # ACCUMULATE alone leaves the codes
    # the selection, given the GPU's P
    mask, cnt = F.falqon_proxy_update(w, dev_f32([s_w]), p, None, None, flags=F.PROXY_SELECT, dev_status=st)
    torch.cuda.synchronize()
    rw, rp, rmask, rcnt = O.proxy_select(wq, s_w, Pg)
    assert rcnt > 0
    np.testing.assert_array_equal(host(mask), rmask)
    assert int(host(cnt)[0]) == rcnt
    np.testing.assert_array_equal(host(w), rw)
    np.testing.assert_array_equal(host(p).view(np.uint32), rp.view(np.uint32))
    assert int(st.item()) == 0


def test_tensor_accumulation_with_both_flags_equals_two_calls(cuda_device):
    N, K, r = 256, 512, 512
    wq, s_w, P, dB, A = _case(5, N, K, r)
    w1, p1 = dev_u8(wq), dev_f32(P)
    w2, p2 = dev_u8(wq), dev_f32(P)
    s = dev_f32([s_w])
    m1, c1 = F.falqon_proxy_update(w1, s, p1, dev_bf16(dB), dev_bf16(A),
                                   flags=F.PROXY_ACCUMULATE | F.PROXY_SELECT | F.PROXY_TENSOR)
    F.falqon_proxy_update(w2, s, p2, dev_bf16(dB), dev_bf16(A), flags=F.PROXY_ACCUMULATE | F.PROXY_TENSOR)
    m2, c2 = F.falqon_proxy_update(w2, s, p2, None, None, flags=F.PROXY_SELECT)
    torch.cuda.synchronize()
    assert torch.equal(m1, m2) and int(c1.item()) == int(c2.item())
    assert torch.equal(w1, w2) and torch.equal(p1.view(torch.int32), p2.view(torch.int32))
