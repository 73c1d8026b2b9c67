"""Seeded synthetic inputs and the named layer shapes.

This module is shared by the CPU oracle (``oracle/``) and by the CUDA path
(``padding_free_moe_b200``).  It holds shapes, random draws and dtype rounding
only: none of the layer's arithmetic (no gating, no sorting, no expert maths).
"""
from .configs import CONFIGS, LayerConfig, get_config, small_configs  # noqa: F401
from .generate import LayerInputs, make_inputs  # noqa: F401
