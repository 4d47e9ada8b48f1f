"""Separate LoRA paths (C-17, the comparison FALQON is measured against) on
the GPU against the oracle.

Each stage is checked given the GPU's previous intermediate (S, then G):
S and G against the oracle's float64 products (C-12); in the FP8 path the
codes and scales of A, B, S and G bit-exact against the oracle's
quantization of the same tensors; Y and dX, which add the adapter branch to
the backbone output as bf16 tensors add, within one bf16 unit of each
branch and of the sum (branch_sum_report); dB and dA against the float64
products of the GPU's S and G (C-12)."""

import numpy as np
import pytest
import torch

import fp8_quantized_lora_b200 as F
import oracle as O
from gpu_util import dev_bf16, dev_f32, dev_u8, host, host_bf16_bits, status_word
from oracle import separate as SP
from oracle.tolerance import branch_sum_report
from synthetic import gen

pytestmark = pytest.mark.gpu


def _inputs(seed, M, N, K, r):
    X = gen.normal_bf16_bits(seed, (M, K), 1.0)
    W = gen.normal_f32(seed + 1, (N, K), 0.02)
    A = gen.normal_bf16_bits(seed + 2, (r, K), 0.01)
    B = gen.normal_bf16_bits(seed + 3, (N, r), 0.01)
    dY = gen.normal_bf16_bits(seed + 4, (M, N), 1e-3)
    wq, s_w, _, _ = O.quantize(W)
    xq, s_x, _, _ = O.quantize(X)
    dyq, s_dy, _, _ = O.quantize(dY)
    return dict(X=X, A=A, B=B, dY=dY, wq=wq, s_w=s_w, xq=xq, s_x=s_x, dyq=dyq, s_dy=s_dy)


def _ok(rep, what):
    assert rep["ok"], (what, rep)


@pytest.mark.parametrize("precision", [F.SEPARATE_BF16, F.SEPARATE_FP8])
@pytest.mark.parametrize("M,N,K,r", [
    (256, 512, 512, 16),
    (200, 272, 336, 32),     # ragged: no dimension a multiple of the tiles
    (1024, 768, 1024, 64),
    (512, 512, 256, 256),    # r above one 256-wide output tile
])
def test_separate_path_matches_oracle(cuda_device, precision, M, N, K, r):
    O.set_threads(16)
    c = _inputs(M + N + K + r, M, N, K, r)
    name = "fp8" if precision == F.SEPARATE_FP8 else "bf16"
    d = {k: (dev_u8(v) if v.dtype == np.uint8 else dev_bf16(v)) for k, v in c.items()
         if isinstance(v, np.ndarray)}
    s_x, s_w, s_dy = dev_f32([c["s_x"]]), dev_f32([c["s_w"]]), dev_f32([c["s_dy"]])
    st = status_word()
    y, saved = F.falqon_lora_separate_fwd(precision, d["xq"], s_x, d["X"], d["wq"], s_w, d["A"], d["B"],
                                          dev_status=st)
    sv = F.separate_saved_views(saved, precision, M, N, K, r)
    qws = F.falqon_workspace_size(F.OP_QUANTIZE, 1, 16)
    bop = F.OP_SEPARATE_BWD_FP8 if precision == F.SEPARATE_FP8 else F.OP_SEPARATE_BWD_BF16
    ws = F.workspace(bop, M, N, K, r, device="cuda:0")
    dx, dA, dB = F.falqon_lora_separate_bwd(precision, d["dyq"], s_dy, d["dY"], d["wq"], s_w, d["xq"], s_x, d["X"],
                                            d["A"], d["B"], saved, dev_status=st, workspace=ws)
    bv = F.separate_bwd_views(ws, precision, M, N, r, qws)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    S_gpu = O.bf16_to_f64(host_bf16_bits(sv["S"]))
    G_gpu = O.bf16_to_f64(host_bf16_bits(bv["G"]))

    exact = SP.separate_fwd(c["X"], c["A"], c["B"], c["xq"], c["s_x"], c["wq"], c["s_w"], name, rnd=False)
    _ok(O.tolerance_report(host_bf16_bits(sv["S"]), exact["S"]), "S")
    f = SP.separate_fwd(c["X"], c["A"], c["B"], c["xq"], c["s_x"], c["wq"], c["s_w"], name, S_given=S_gpu)
    if precision == F.SEPARATE_FP8:
        sc = host(sv["scales"])
        assert sc[1] == f["s_a"] and sc[2] == f["s_b"] and sc[0] == f["s_s"]
        np.testing.assert_array_equal(host(sv["aq"]), f["aq"])
        np.testing.assert_array_equal(host(sv["bq"]), f["bq"])
        np.testing.assert_array_equal(host(sv["sq"]), f["sq"])
    _ok(branch_sum_report(host_bf16_bits(y), f["Y"], [f["Ybb"], f["Ylora"]]), "Y")

    ex_b = SP.separate_bwd(c["X"], c["dY"], c["A"], c["B"], S_gpu, c["xq"], c["s_x"], c["dyq"], c["s_dy"], c["wq"],
                           c["s_w"], name, rnd=False)
    _ok(O.tolerance_report(host_bf16_bits(bv["G"]), ex_b["G"]), "G")
    b = SP.separate_bwd(c["X"], c["dY"], c["A"], c["B"], S_gpu, c["xq"], c["s_x"], c["dyq"], c["s_dy"], c["wq"],
                        c["s_w"], name, G_given=G_gpu)
    if precision == F.SEPARATE_FP8:
        assert float(host(bv["s_g"])[0]) == b["s_g"]
        np.testing.assert_array_equal(host(bv["gq"]), b["gq"])
    _ok(branch_sum_report(host_bf16_bits(dx), b["dX"], [b["dXbb"], b["dXlora"]]), "dX")
    ex_g = SP.separate_bwd(c["X"], c["dY"], c["A"], c["B"], S_gpu, c["xq"], c["s_x"], c["dyq"], c["s_dy"], c["wq"],
                           c["s_w"], name, G_given=G_gpu, rnd=False)
    _ok(O.tolerance_report(host_bf16_bits(dB), ex_g["dB"]), "dB")
    _ok(O.tolerance_report(host_bf16_bits(dA), ex_g["dA"]), "dA")


@pytest.mark.parametrize("precision", [F.SEPARATE_BF16, F.SEPARATE_FP8])
def test_separate_output_subsets(cuda_device, precision):
    """dB alone and dA alone equal the corresponding outputs of a full call."""
    M, N, K, r = 256, 256, 256, 32
    c = _inputs(77, M, N, K, r)
    d = {k: (dev_u8(v) if v.dtype == np.uint8 else dev_bf16(v)) for k, v in c.items() if isinstance(v, np.ndarray)}
    s_x, s_w, s_dy = dev_f32([c["s_x"]]), dev_f32([c["s_w"]]), dev_f32([c["s_dy"]])
    _, saved = F.falqon_lora_separate_fwd(precision, d["xq"], s_x, d["X"], d["wq"], s_w, d["A"], d["B"])
    args = (precision, d["dyq"], s_dy, d["dY"], d["wq"], s_w, d["xq"], s_x, d["X"], d["A"], d["B"], saved)
    full = F.falqon_lora_separate_bwd(*args)
    only_db = F.falqon_lora_separate_bwd(*args, dx=None, dA=None)
    only_da = F.falqon_lora_separate_bwd(*args, dx=None, dB=None)
    torch.cuda.synchronize()
    assert only_db[0] is None and only_db[1] is None and only_da[2] is None
    np.testing.assert_array_equal(host_bf16_bits(only_db[2]), host_bf16_bits(full[2]))
    np.testing.assert_array_equal(host_bf16_bits(only_da[1]), host_bf16_bits(full[1]))
