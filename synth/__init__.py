"""Seeded synthetic inputs for the Ideogram 4 DiT block and stack.

This package is shared by the CPU oracle's tests and by the CUDA path's tests
and benchmark, and holds none of the block's arithmetic: it only draws numbers
(one numpy ``default_rng`` stream per tensor, keyed by (seed, block, name)),
rounds them to the storage type (bf16, or FP8 E4M3 with a per-output-channel
fp32 scale for the release-precision weights) and names the workload shapes.
Both sides consume exactly the rounded values, so input rounding is never part
of a parity error.
"""

from .configs import CONFIGS, Config, get_config  # noqa: F401
from .block_inputs import (  # noqa: F401
    make_block_weights,
    make_block_weights_device,
    make_block_activations,
    make_stack_inputs,
    make_text_cond_inputs,
    quantize_e4m3_per_channel,
    tensor_rng,
)
