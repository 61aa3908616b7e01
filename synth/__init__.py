"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

Holds no arithmetic of the method itself; see :mod:`synth.workloads`.
"""
from .workloads import (  # noqa: F401
    BLK,
    CONFIGS,
    Workload,
    chunk_seed,
    chunk_tokens,
    coverage,
    direct_blocks,
    prior,
    random_bf16,
)
from .geometry import SlabScene, slab_scene  # noqa: F401
