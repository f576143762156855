"""Seeded synthetic inputs for the Star Attention hot path.

This package holds no step of the method's arithmetic: it only draws the
Q/K/V tensors, position ids and the peaky-key selection that both the CUDA
path (through the tests and ``bench.py``) and the CPU oracle consume.

* :mod:`synth.gen`      -- the counter-based generator (SplitMix64 + Box-Muller).
* :mod:`synth.configs`  -- the named workloads (shapes, block sizes, value mix).
"""

from .configs import CONFIGS, Workload, get_config  # noqa: F401
from .gen import (  # noqa: F401
    STREAM_IDS,
    gaussian_bf16,
    layer_inputs,
    make_inputs,
    peaky_rows,
    splitmix64_reference,
    uniform_pair_u64,
)
