"""Seeded synthetic inputs for the SVDQuant W4A4 linear layer.

This module only draws numbers. It holds none of the method's arithmetic
(no smoothing, no SVD, no quantisation): it produces the activations X, the
weights W and the bias that both the CPU oracle and the CUDA path consume,
so that the two sides see bit-identical inputs.

Recipe (stated once here, used everywhere):

* random bits: SplitMix64 evaluated at counter i of stream s, i.e. the
  published SplitMix64 finaliser applied to ``seed(s) + (i + 1) * 0x9E3779B97F4A7C15``;
* uniforms: the top 53 bits of a SplitMix64 word, scaled by 2^-53, in [0, 1);
* normals: Box-Muller in fp64 on consecutive uniform pairs;
* every bf16 tensor: the fp64 sample rounded once, to nearest-even, to bf16.

Workloads follow the layer shapes of a 12B-parameter FLUX.1 DiT (hidden 3072,
4096 image + 512 text tokens), which the SVDQuant pages use as their flagship
model (ai-digest.ru "SVDQuant: absorbing outliers ...", abstract). No dataset
or trained weight is used: distributions below stand in for them.
"""

from .generator import (  # noqa: F401
    SplitMix64Stream,
    bf16_bits_from_f64,
    bf16_bits_to_f32,
    normal,
    uniform,
)
from .workloads import (  # noqa: F401
    CONFIGS,
    LayerInputs,
    make_layer_inputs,
    make_activation,
    make_lora,
    make_stack_layer_inputs,
    make_weight,
    stack_layer_shapes,
)
