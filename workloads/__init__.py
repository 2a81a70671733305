"""Seeded synthetic decode workloads shaped like the Loki evaluation settings.

This package only draws random inputs (keys, values, queries, calibration keys)
and describes workload shapes.  It contains none of the attention method's
arithmetic: no PCA, no rotation, no scoring, no selection, no softmax.  Both the
CUDA path (through its tests and the benchmark) and the fp64 oracle consume the
arrays produced here.
"""
from .configs import WORKLOADS, Workload, get_workload, mistral_sweep_points
from .generators import (
    KeyModel,
    make_key_model,
    draw_keys,
    draw_normal,
    to_cache_dtype,
    decode_inputs,
)

__all__ = [
    "WORKLOADS",
    "Workload",
    "get_workload",
    "mistral_sweep_points",
    "KeyModel",
    "make_key_model",
    "draw_keys",
    "draw_normal",
    "to_cache_dtype",
    "decode_inputs",
]
