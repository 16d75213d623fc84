"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This package holds model shapes, a counter-based weight generator and prompt
generators.  It contains none of the decoding method's arithmetic: it only
produces the numbers both implementations consume.  Every value it returns is
a pure function of (seed, tensor name, element index), so the same weights come
out bit for bit on the CPU and on a GPU.
"""
from .configs import ModelDims, SpecConfig, CONFIGS, get_config, tap_layers_evenly
from .weights import (weight_names, weight_shapes, make_weight, make_weights,
                      hash32, centered_irwin_hall)
from .prompts import zipf_prompt, uniform_prompt, make_prompt

__all__ = [
    "ModelDims", "SpecConfig", "CONFIGS", "get_config", "tap_layers_evenly",
    "weight_names", "weight_shapes", "make_weight", "make_weights",
    "hash32", "centered_irwin_hall", "zipf_prompt", "uniform_prompt", "make_prompt",
]
