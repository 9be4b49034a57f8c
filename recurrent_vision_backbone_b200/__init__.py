"""GTR token-mixer forward pass (key-decay gated linear attention) for B200.

The compute path is the CUDA library ``libgtr_gla.so`` (C ABI in
``include/gtr_gla.h``); ``recurrent_vision_backbone_b200.gla`` is its Python
binding and ``recurrent_vision_backbone_b200.inputs`` the seeded input recipe.
Nothing is loaded at import time.
"""
__all__ = ["gla", "inputs", "build"]
