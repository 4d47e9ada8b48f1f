"""falqon_quantize on the GPU against the oracle: bit-exact codes, scales,
amax, residuals and status bits."""

import numpy as np
import pytest
import torch

import fp8_quantized_lora_b200 as F
import oracle as O
from gpu_util import dev_bf16, dev_f32, host, status_word
from synthetic import WORKLOADS, gen, layer_inputs

pytestmark = pytest.mark.gpu


def _run(x_np, residual=False):
    x = dev_bf16(x_np) if x_np.dtype == np.uint16 else dev_f32(x_np)
    st = status_word()
    res = torch.empty(x.shape, dtype=torch.float32, device=x.device) if residual else None
    codes, s, a = F.falqon_quantize(x, residual=res, dev_status=st)
    torch.cuda.synchronize()
    return host(codes), np.float32(host(s)[0]), np.float32(host(a)[0]), int(host(st)[0]), (
        host(res) if residual else None)


def _check(x_np, residual=False):
    codes, s, a, st, res = _run(x_np, residual)
    rc, rs, ra, rst = O.quantize(x_np)
    assert st == rst
    assert s.view(np.uint32) == rs.view(np.uint32), (s, rs)
    assert a.view(np.uint32) == ra.view(np.uint32), (a, ra)
    np.testing.assert_array_equal(codes, rc)
    if residual:
        _, r32 = O.residual(x_np, rc, rs)
        np.testing.assert_array_equal(res.view(np.uint32), r32.view(np.uint32))


# up to 2^20 elements the library takes the two-launch path (amax partials,
# then the cast); above it the cooperative one-launch stream kernel
@pytest.mark.parametrize("shape", [(256, 512), (1, 16), (37, 48), (129, 272), (1000, 1008), (1024, 1024),
                                   (1031, 1040), (4097, 272), (2048, 2064)])
def test_bf16_activations(cuda_device, shape):
    _check(gen.normal_bf16_bits(11 + shape[0], shape, 1.0))


@pytest.mark.parametrize("shape", [(512, 512), (37, 48), (300, 4096), (257, 4112)])
def test_f32_weights_with_eq8_residual(cuda_device, shape):
    _check(gen.normal_f32(21 + shape[0], shape, 0.02), residual=True)


def test_gradient_scale_and_tiny_values(cuda_device):
    _check(gen.normal_bf16_bits(31, (64, 128), 1e-3))
    _check(gen.normal_bf16_bits(32, (64, 128), 1e-30))


def test_llama_attention_activation_full_size(cuda_device):
    wl = WORKLOADS["llama7b_attn_proj_4096x4096x4096_r64"]
    d = layer_inputs(wl, wl.layers[0])
    _check(d["X"])
    _check(d["dY"])
    _check(d["W"], residual=True)


def test_llama_mlp_down_activation_full_size(cuda_device):
    # 8192 x 11008: larger than L2, so the cast pass re-reads from HBM
    _check(gen.normal_bf16_bits(41, (8192, 11008), 1.0))


def test_all_zero_and_single_element(cuda_device):
    _check(np.zeros((16, 32), dtype=np.uint16))
    x = np.zeros((16, 32), dtype=np.float32)
    x[5, 17] = -3.0
    codes, s, a, st, _ = _run(x)
    assert codes[5, 17] == 0xFE and np.count_nonzero(codes) == 1 and st == 0


def test_nonfinite_input_sets_status(cuda_device):
    x = gen.normal_bf16_bits(51, (32, 64), 1.0)
    x[3, 3] = 0x7FC0  # NaN
    codes, s, a, st, _ = _run(x)
    assert st & F.DEV_NONFINITE and s == 1.0 and not np.isfinite(a)
    x[3, 3] = 0x7F80  # +inf
    codes, s, a, st, _ = _run(x)
    assert st & F.DEV_NONFINITE and s == 1.0 and np.isinf(a)


def test_scale_overflow_sets_status(cuda_device):
    x = np.zeros((16, 16), dtype=np.float32)
    x[0, 0] = 1e-39  # 448 / 1e-39 overflows float32
    _check(x)
    codes, s, a, st, _ = _run(x)
    assert st & F.DEV_SCALE_OVERFLOW and s == np.finfo(np.float32).max


def test_all_bf16_patterns_encode_like_the_oracle(cuda_device):
    # every bf16 bit pattern with |x| <= 448, with 448 present so the scale is exactly 1
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = gen.bf16_bits_to_f32(b)
    keep = np.isfinite(f) & (np.abs(f) <= 448)
    x = np.concatenate([b[keep], gen.f32_to_bf16_bits(np.float32([448.0]))])
    x = np.concatenate([x, np.zeros((-len(x)) % 16, dtype=np.uint16)]).reshape(-1, 16)
    codes, s, _, _, _ = _run(x)
    assert s == 1.0
    np.testing.assert_array_equal(codes, O.e4m3_encode(gen.bf16_bits_to_f32(x)))


def test_fp32_patterns_encode_like_the_oracle(cuda_device):
    # a prime-stride sweep over the float32 patterns with |x| <= 448 (both signs)
    top = np.uint32(0x43E00000)  # 448.0
    pats = (np.arange(0, 1 << 25, dtype=np.uint64) * np.uint64(67) % np.uint64(int(top) + 1))
    pats = pats.astype(np.uint32)
    sign = (np.arange(len(pats)) & 1).astype(np.uint32) << np.uint32(31)
    f = (pats | sign).view(np.float32)
    f = np.concatenate([f, np.float32([448.0])])
    f = np.concatenate([f, np.zeros((-len(f)) % 1024, dtype=np.float32)]).reshape(-1, 1024)
    codes, s, _, _, _ = _run(f)
    assert s == 1.0
    np.testing.assert_array_equal(codes, O.e4m3_encode(f))


def test_every_fp32_pattern_up_to_448_encodes_like_the_oracle(cuda_device):
    """Exhaustive: every float32 bit pattern from +0 to 448 (1.14e9 values),
    quantized on the GPU in chunks that each hold 448 (so s = 1 exactly),
    against the oracle's encoder; the negative patterns are checked by the
    format's sign symmetry (the code of -x is the code of x with bit 7 set)."""
    from concurrent.futures import ThreadPoolExecutor

    top = 0x43E00000  # 448.0
    chunk = 1 << 27
    dev = torch.device("cuda:0")
    st = status_word()
    ws = F.workspace(F.OP_QUANTIZE, 1, chunk + 16, device=dev)  # initialised once, reused by every call
    pool = ThreadPoolExecutor(max_workers=16)

    def oracle_codes(f):
        parts = np.array_split(f, 16)
        return np.concatenate(list(pool.map(O.e4m3_encode, parts)))

    for lo in range(0, top + 1, chunk):
        hi = min(top + 1, lo + chunk)
        pats = np.arange(lo, hi, dtype=np.uint32)
        n = len(pats) + 1
        pad = (-n) % 16
        f = np.concatenate([pats.view(np.float32), np.float32([448.0]), np.zeros(pad, np.float32)])
        x = torch.from_numpy(f).to(dev)
        codes, s, _ = F.falqon_quantize(x.view(-1, 16), dev_status=st, workspace=ws)
        neg, s_neg, _ = F.falqon_quantize((-x).view(-1, 16), dev_status=st, workspace=ws)
        torch.cuda.synchronize()
        assert float(s.item()) == 1.0 and float(s_neg.item()) == 1.0
        assert torch.equal(neg.view(-1)[: len(pats)], codes.view(-1)[: len(pats)] | 0x80), hex(lo)
        np.testing.assert_array_equal(host(codes).reshape(-1)[: len(pats)], oracle_codes(pats.view(np.float32)),
                                      err_msg=hex(lo))
    pool.shutdown()
    assert int(st.item()) == 0


def test_one_workspace_reused_across_sizes_and_graph_replays(cuda_device):
    """The workspace contract: initialised once, then reused by calls of both
    paths (small tensors take the two-launch path, large ones the exchange
    with its generation counter) and by replays of a captured graph; every
    call's scale and codes equal the oracle's."""
    dev = torch.device("cuda:0")
    ws = F.workspace(F.OP_QUANTIZE, 1, 16, device=dev)
    st = status_word()
    shapes = [(4096, 1024), (64, 64), (2048, 2048), (4096, 1024), (512, 512), (8192, 512)]
    for i, shape in enumerate(shapes):
        x = gen.normal_bf16_bits(500 + i, shape, 10.0 ** (i % 3 - 1))
        codes, s, _ = F.falqon_quantize(dev_bf16(x), dev_status=st, workspace=ws)
        rc, rs, _, _ = O.quantize(x)
        torch.cuda.synchronize()
        assert float(s.item()) == float(rs), shape
        np.testing.assert_array_equal(host(codes), rc)
    # a captured quantize replayed on changing data reuses the same workspace words
    xs = dev_bf16(gen.normal_bf16_bits(600, (4096, 1024), 1.0))
    codes = torch.empty(xs.shape, dtype=torch.uint8, device=dev)
    scale = torch.empty(1, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        F.falqon_quantize(xs, codes=codes, scale=scale, dev_status=st, workspace=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        F.falqon_quantize(xs, codes=codes, scale=scale, dev_status=st, workspace=ws)
    for k in range(5):
        x = gen.normal_bf16_bits(700 + k, (4096, 1024), 2.0 ** (k - 2))
        xs.copy_(dev_bf16(x))
        g.replay()
        torch.cuda.synchronize()
        rc, rs, _, _ = O.quantize(x)
        assert float(scale.item()) == float(rs), k
        np.testing.assert_array_equal(host(codes), rc)
    assert int(st.item()) == 0
