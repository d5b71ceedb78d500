"""Seeded synthetic inputs for chunked-prefill block-sparse attention.

This package holds only input generation: workload shapes, seeded Q/K/V
pages, page permutations and 2D block-sparse masks.  It contains none of the
method's arithmetic (no union, no compaction, no attention); both the CUDA
path and the float64 oracle consume what it produces.
"""
from .configs import CONFIGS, Workload, get_config, sweep_chunk, density_cell  # noqa: F401
from .generators import (  # noqa: F401
    make_qkv_pages,
    bernoulli_mask,
    vertical_slash_mask,
    ones_mask,
    pack_mask_bits,
    mask_for,
    causal_live,
    last_live_block,
    quantize_pages_e4m3,
)
