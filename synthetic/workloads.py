"""Workload shapes and input recipes for the melded FP8 linear step.

The shapes follow the LLaMA-7B fine-tuning layers the FALQON pages train on
(LLaMA-7B/13B, OpenReview rebuttal, "W3.1" and the experiments with rank 64,
"Q2" of the third reviewer): hidden size 4096, MLP width 11008, adapter rank
16-8192.  No dataset or checkpoint is involved; every tensor is a seeded
normal draw (see ``gen``), with the standard deviations listed per workload.

Tensor names and layouts (all row-major):
  X   [M, K]  activations, bfloat16
  W   [N, K]  high-precision weight, float32 (quantized once to Wq)
  A   [r, K]  adapter down-projection, bfloat16 (frozen, LoRA-FA style)
  B   [N, r]  adapter up-projection, bfloat16 (zero at step 0)
  dY  [M, N]  output gradient, bfloat16
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import gen


@dataclass(frozen=True)
class Layer:
    name: str
    K: int          # in features
    N: int          # out features
    x_group: str    # layers with the same x_group share one activation X


@dataclass(frozen=True)
class Workload:
    name: str
    M: int
    r: int
    layers: tuple
    n_stack: int = 1          # number of transformer blocks (repeats of ``layers``)
    x_std: float = 1.0
    w_std: float = 0.02
    a_std: float = 0.01
    dy_std: float = 1e-3
    lr: float = 1e-3          # plain SGD step on B; the proxy receives dB_inc = -lr * dB
    seed: int = 0
    description: str = ""
    ranks: tuple = field(default=())


_ATTN = (Layer("proj", 4096, 4096, "x"),)
_MLP = (Layer("gate", 4096, 11008, "x_mlp"), Layer("up", 4096, 11008, "x_mlp"),
        Layer("down", 11008, 4096, "x_down"))
_BLOCK = (Layer("q", 4096, 4096, "x_attn"), Layer("k", 4096, 4096, "x_attn"),
          Layer("v", 4096, 4096, "x_attn"), Layer("o", 4096, 4096, "x_o"),
          Layer("gate", 4096, 11008, "x_mlp"), Layer("up", 4096, 11008, "x_mlp"),
          Layer("down", 11008, 4096, "x_down"))

WORKLOADS = {
    "tiny_256x512x512_r16": Workload(
        "tiny_256x512x512_r16", M=256, r=16, layers=(Layer("proj", 512, 512, "x"),),
        dy_std=1e-2, lr=1.0,
        description="single linear layer, M=256 K=512 N=512 r=16, seed 0"),
    "llama7b_attn_proj_4096x4096x4096_r64": Workload(
        "llama7b_attn_proj_4096x4096x4096_r64", M=4096, r=64, layers=_ATTN,
        description="LLaMA-7B attention projection: M=4096 tokens (4 x 1024), K=N=4096, r=64"),
    "llama7b_mlp_8192tok_r64": Workload(
        "llama7b_mlp_8192tok_r64", M=8192, r=64, layers=_MLP,
        description="LLaMA-7B MLP gate/up 4096->11008 and down 11008->4096, M=8192 tokens, r=64"),
    "llama2_7b_stack_32x7_4096tok_r16": Workload(
        "llama2_7b_stack_32x7_4096tok_r16", M=4096, r=16, layers=_BLOCK, n_stack=32,
        description="32 blocks x {q,k,v,o,gate,up,down}, M=8x512 tokens, r=16"),
    "rank_sweep_4096cube": Workload(
        "rank_sweep_4096cube", M=4096, r=64, layers=_ATTN,
        ranks=(16, 64, 256, 1024, 4096, 8192),
        description="adapter-rank sweep at M=K=N=4096"),
}


def layer_inputs(wl: Workload, layer: Layer, step: int = 0, block: int = 0,
                 r: int | None = None, with_b: bool = False) -> dict:
    """Seeded inputs for one layer of one step.

    X and dY are fresh per step; W and A are fixed per (block, layer); B is
    zero at step 0 unless ``with_b`` asks for a nonzero draw (std 1e-3), which
    the parity tests use to exercise the dA path.
    """
    r = wl.r if r is None else r
    tag = f"{wl.name}/b{block}/{layer.name}"
    xtag = f"{wl.name}/b{block}/{layer.x_group}/step{step}"
    s = wl.seed
    out = {
        "X": gen.normal_bf16_bits(gen.stream_seed(s, xtag + "/X"), (wl.M, layer.K), wl.x_std),
        "W": gen.normal_f32(gen.stream_seed(s, tag + "/W"), (layer.N, layer.K), wl.w_std),
        "A": gen.normal_bf16_bits(gen.stream_seed(s, tag + f"/A/r{r}"), (r, layer.K), wl.a_std),
        "dY": gen.normal_bf16_bits(gen.stream_seed(s, tag + f"/dY/step{step}"), (wl.M, layer.N),
                                   wl.dy_std),
    }
    if with_b:
        out["B"] = gen.normal_bf16_bits(gen.stream_seed(s, tag + f"/B/r{r}"), (layer.N, r), 1e-3)
    else:
        out["B"] = np.zeros((layer.N, r), dtype=np.uint16)
    return out
