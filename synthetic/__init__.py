"""Seeded synthetic inputs for the melded FP8 linear step.

This package holds the input generators and the workload shapes, and none of
the method's arithmetic: no quantization, no scaling, no GEMM.  Both the CPU
oracle (through the tests) and the CUDA path (through the tests and the bench)
draw their inputs from here, so that the two sides see identical bytes.

Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) used in counter mode, i.e. the i-th draw of a
stream seeded with ``s`` is ``mix64(s + (i + 1) * 0x9E3779B97F4A7C15)``; two
uniform draws feed one Box-Muller pair.  Normal draws are made in float64,
scaled by the requested standard deviation, rounded to float32 (round to
nearest even), and, for bfloat16 tensors, rounded once more to bfloat16
(round to nearest even on the float32 bit pattern).
"""

from .gen import (  # noqa: F401
    GOLDEN_GAMMA,
    splitmix64,
    stream_seed,
    uniform01,
    normal,
    normal_f32,
    normal_bf16_bits,
    f32_to_bf16_bits,
    bf16_bits_to_f32,
)
from .workloads import WORKLOADS, Workload, layer_inputs  # noqa: F401
