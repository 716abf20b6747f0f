"""Seeded synthetic workloads for the paged decode step, the host allocator
model that hands out their block tables, and the algorithmic byte model.

Shared by the tests, the benchmark and the oracle's callers; contains none
of the attention, cache-write or block-copy arithmetic itself.
"""
from . import block_manager, byte_model, generators  # noqa: F401
from .block_manager import BlockManager  # noqa: F401
from .generators import CONFIGS, DecodeWorkload  # noqa: F401
