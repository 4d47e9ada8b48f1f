"""Failure detection on the GPU without a fault: the library's bounded waits
(an mbarrier wait as in the tcgen05 and quantize kernels, and a bounded poll
as in the quantize kernel's grid exchange) run out on things that never
complete, report FALQON_DEV_TIMEOUT through the status word, and leave the
context usable for the next call."""

import numpy as np
import pytest
import torch

import fp8_quantized_lora_b200 as F
import oracle as O
from gpu_util import dev_bf16, host, status_word
from synthetic import gen

pytestmark = pytest.mark.gpu


def _selftest(flag_value):
    dev = torch.device("cuda:0")
    flag = torch.full((1,), flag_value, dtype=torch.int32, device=dev)
    st, which = status_word(), torch.zeros(1, dtype=torch.int32, device=dev)
    F.falqon_selftest_bounded_waits(flag, st, which)
    torch.cuda.synchronize()
    return int(st.item()), int(which.item())


def test_waits_that_cannot_complete_report_a_timeout(cuda_device):
    st, which = _selftest(0)
    assert st == F.DEV_TIMEOUT and which == 3  # both waits gave up
    st, which = _selftest(1)
    assert st == F.DEV_TIMEOUT and which == 1  # the poll saw its flag; the mbarrier wait still gave up


def test_the_context_stays_usable_after_a_timeout(cuda_device):
    _selftest(0)
    x = gen.normal_bf16_bits(5, (64, 128), 1.0)
    st = status_word()
    codes, s, _ = F.falqon_quantize(dev_bf16(x), dev_status=st)
    torch.cuda.synchronize()
    rc, rs, _, _ = O.quantize(x)
    assert int(st.item()) == 0
    assert np.array_equal(host(codes), rc) and host(s)[0] == rs
