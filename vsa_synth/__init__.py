"""Seeded synthetic inputs for the tile-sparse attention layer.

This module is the one piece shared by the fp64 oracle and the CUDA path:
it only draws numbers and lays them out. It holds none of the method's
arithmetic (no tiling, pooling, scoring, selection or attention).

Random numbers come from SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast
splittable pseudorandom number generators", OOPSLA 2014; the 64-bit
finaliser as published by S. Vigna), used counter-style: output i of the
generator seeded with ``s`` is ``mix(s + (i + 1) * GAMMA)``. Normals use the
Box-Muller transform (cos branch) on two consecutive outputs.

Every tensor the layer consumes is produced here once, rounded to bf16
(round-to-nearest-even from fp32), and handed to both sides as the same
bytes.
"""
from .generate import (  # noqa: F401
    GAMMA,
    splitmix64_outputs,
    uniform01,
    standard_normal,
    f32_to_bf16_bits,
    bf16_bits_to_f32,
    position_embedding,
    LayerInputs,
    make_layer_inputs,
)
from .configs import CONFIGS, LayerConfig, get_config  # noqa: F401
