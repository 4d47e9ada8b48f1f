"""The grouped forward (layers that read one quantized activation, in one
launch) against falqon_linear_fwd on the same operands (bit-identical: the
same arithmetic) and against the oracle (C-5 within C-12)."""

import numpy as np
import pytest
import torch

import fp8_quantized_lora_b200 as F
import oracle as O
from gpu_util import dev_bf16, dev_f32, dev_u8, host_bf16_bits, status_word
from synthetic import gen

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,Ns", [
    (256, 512, (512, 512, 512)),      # q | k | v
    (200, 336, (1008, 1008)),         # gate | up, ragged rows and widths
    (300, 256, (272, 16, 784)),       # uneven segments, one narrower than a tile
    (128, 512, (1024,)),              # one segment
])
def test_grouped_forward(cuda_device, M, K, Ns):
    O.set_threads(16)
    xq, s_x, _, _ = O.quantize(gen.normal_bf16_bits(M + K, (M, K), 1.0))
    ws = [O.quantize(gen.normal_f32(M + K + 10 * i, (n, K), 0.02))[:2] for i, n in enumerate(Ns)]
    x_d, sx_d = dev_u8(xq), dev_f32([s_x])
    wq_d = [dev_u8(w) for w, _ in ws]
    sw_d = [dev_f32([s]) for _, s in ws]
    st = status_word()
    ys = F.falqon_linear_fwd_grouped(x_d, sx_d, wq_d, sw_d, dev_status=st)
    singles = [F.falqon_linear_fwd(x_d, sx_d, w, s) for w, s in zip(wq_d, sw_d)]
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for i, (y, y1) in enumerate(zip(ys, singles)):
        np.testing.assert_array_equal(host_bf16_bits(y), host_bf16_bits(y1), err_msg=f"segment {i}")
    rep = O.tolerance_report(host_bf16_bits(ys[-1]), O.linear_fwd(xq, s_x, ws[-1][0], ws[-1][1]))
    assert rep["ok"], rep
