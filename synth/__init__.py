"""Seeded synthetic inputs for the Sparse Delta Memory forward pass.

This package holds the workload recipes and a counter-based random generator.
It contains none of the method's arithmetic: it only draws q', k', v, the gates,
the codebooks and the initial table M_0.  Both the CUDA path's tests/benchmark
and the CPU oracle take their inputs from here.
"""
from .generate import (  # noqa: F401
    SDMConfig, CONFIGS, config, gen_inputs, gen_head_inputs, gen_gdn_inputs, gen_decay_rate,
    splitmix64_stream,
    uniform01, std_normal,
)
