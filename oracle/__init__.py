"""The oracle: a plain fp64 CPU statement of the Prism Attention decode step.

TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU-baseline leg of the
benchmark).  Independent of the CUDA library: neither imports the other.
"""
from .prism_ref import (CHAIN_ANCHOR, CHAIN_PREV, MODE_DENSE_ANCHOR, MODE_POOL, MODE_REFINE,
                        MODE_STATIC_REUSE, PLANTS, Oracle, bf16_bits, load)

__all__ = ["Oracle", "load", "bf16_bits", "PLANTS", "MODE_REFINE", "MODE_STATIC_REUSE",
           "MODE_DENSE_ANCHOR", "MODE_POOL", "CHAIN_PREV", "CHAIN_ANCHOR"]
