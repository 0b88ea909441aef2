"""Seeded synthetic workloads for the top-k MoE FFN layer.

This package is shared by the CUDA path's tests and benchmark and by the fp64
oracle.  It only draws random tensors and loads stored calibration numbers; it
holds none of the layer's arithmetic (no routing, no expert evaluation).
"""

from .configs import CONFIGS, MoEConfig, get_config, scaled  # noqa: F401
from .gen import make_inputs, make_weights, make_activations, expert_ids  # noqa: F401
