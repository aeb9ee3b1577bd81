"""B200-native LatentMoE layer forward pass.

Submodules: ``lmoe`` (Python binding of the C-ABI library ``liblmoe.so``),
``build`` (compiles it for sm_100a), ``workloads`` (seeded synthetic inputs)
and ``costmodel`` (the paper's roofline formulas and algorithmic counts).
Import them explicitly, e.g. ``from mixture_experts_layer_64_b200 import lmoe``.
"""
