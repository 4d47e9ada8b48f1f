"""falqon_linear_bwd_noalloc: the backward call for callers that cannot
allocate device memory (it keeps its intermediates in the library's built-in
scratch array instead of a caller workspace).

Checked through the C ABI against falqon_linear_bwd on the same inputs, on
two calls in a row with different data (the second call must not be affected
by what the first left in the shared scratch), within the float acceptance
rule the other tests use; the kernels are deterministic, so the outputs are
also bit-identical.  Runs alone or after the other tests.
"""

import numpy as np
import pytest
import torch

import fp8_quantized_lora_b200 as F
import oracle as O
from gpu_util import dev_bf16, dev_f32, dev_u8, host_bf16_bits, status_word
from synthetic import gen

pytestmark = pytest.mark.gpu


def _inputs(seed, M, N, K, r):
    xq, s_x, _, _ = O.quantize(gen.normal_bf16_bits(seed, (M, K), 1.0))
    dyq, s_dy, _, _ = O.quantize(gen.normal_bf16_bits(seed + 1, (M, N), 1e-3))
    wq, s_w, _, _ = O.quantize(gen.normal_f32(seed + 2, (N, K), 0.02))
    A = gen.normal_bf16_bits(seed + 3, (r, K), 0.01)
    B = gen.normal_bf16_bits(seed + 4, (N, r), 1e-3)
    return (dev_u8(dyq), dev_f32([s_dy]), dev_u8(wq), dev_f32([s_w]), dev_u8(xq), dev_f32([s_x]),
            dev_bf16(A), dev_bf16(B))


def _same(got, ref):
    g, r = host_bf16_bits(got), host_bf16_bits(ref)
    rf = (r.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    rep = O.tolerance_report(g, rf)
    assert rep["ok"], rep
    np.testing.assert_array_equal(g, r)


@pytest.mark.parametrize("M,N,K,r", [(4096, 4096, 4096, 64), (200, 272, 336, 32)])
def test_noalloc_matches_workspace_entry_point_twice(cuda_device, M, N, K, r):
    for call, seed in enumerate((11, 29)):
        args = _inputs(seed + M, M, N, K, r)
        st1, st2 = status_word(), status_word()
        ref = F.falqon_linear_bwd(*args, dev_status=st1)
        got = F.falqon_linear_bwd_noalloc(*args, dev_status=st2)
        torch.cuda.synchronize()
        assert int(st1.item()) == 0 and int(st2.item()) == 0, call
        for g, rr in zip(got, ref):
            _same(g, rr)


@pytest.mark.parametrize("outputs", ["dx", "dA", "dB", "dA+dB", "dx+dB"])
def test_noalloc_output_subsets_after_a_full_call(cuda_device, outputs):
    """A call asking for only some outputs, right after a full call on other
    data: the half of the shared scratch it does not write still holds the
    first call's values, and must not leak into its results."""
    M, N, K, r = 520, 272, 336, 48
    full = _inputs(101, M, N, K, r)
    F.falqon_linear_bwd_noalloc(*full)
    args = _inputs(202, M, N, K, r)
    want = {k: (k in outputs.split("+")) for k in ("dx", "dA", "dB")}
    st1, st2 = status_word(), status_word()
    ref = F.falqon_linear_bwd(*args, dx=want["dx"], dA=want["dA"], dB=want["dB"], dev_status=st1)
    got = F.falqon_linear_bwd_noalloc(*args, dx=want["dx"], dA=want["dA"], dB=want["dB"], dev_status=st2)
    torch.cuda.synchronize()
    assert int(st1.item()) == 0 and int(st2.item()) == 0
    for name, g, rr in zip(("dx", "dA", "dB"), got, ref):
        assert (g is None) == (not want[name]) and (rr is None) == (not want[name])
        if g is not None:
            _same(g, rr)


def test_noalloc_shape_just_under_the_scratch_limit(cuda_device):
    """M = 32760, r = 64: four planes of 32760 x 64 bf16 take 16 773 120 bytes
    of the 16 777 216-byte scratch (4 KiB short of it)."""
    M, N, K, r = 32760, 256, 256, 64
    need = F.falqon_workspace_size(F.OP_LINEAR_BWD, M, N, K, r)
    assert need == (16 << 20) - 4096
    for seed in (7, 8):
        args = _inputs(seed, M, N, K, r)
        st1, st2 = status_word(), status_word()
        ref = F.falqon_linear_bwd(*args, dev_status=st1)
        got = F.falqon_linear_bwd_noalloc(*args, dev_status=st2)
        torch.cuda.synchronize()
        assert int(st1.item()) == 0 and int(st2.item()) == 0
        for g, rr in zip(got, ref):
            _same(g, rr)


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_device):
    # M = 32768, r = 256 needs far more than the 16 MiB built-in scratch
    M, N, K, r = 32768, 256, 256, 256
    assert F.falqon_workspace_size(F.OP_LINEAR_BWD, M, N, K, r) > 16 << 20
    dev = "cuda:0"
    z8 = torch.zeros((M, N), dtype=torch.uint8, device=dev)
    with pytest.raises(F.FalqonError) as ei:
        F.falqon_linear_bwd_noalloc(z8, torch.ones(1, device=dev), None, None,
                                    torch.zeros((M, K), dtype=torch.uint8, device=dev),
                                    torch.ones(1, device=dev),
                                    torch.zeros((r, K), dtype=torch.bfloat16, device=dev),
                                    torch.zeros((N, r), dtype=torch.bfloat16, device=dev),
                                    dx=None)
    assert ei.value.status == 3  # FALQON_ERR_WORKSPACE, returned before any launch
