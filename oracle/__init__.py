"""CPU oracle of the hashed n-gram embedding lookup -- TEST INFRASTRUCTURE ONLY.

The plain C implementation in ``engram_oracle.c`` (fp64, scalar) is the statement of what
the lookup computes; this module loads it through ctypes.  Only the test suite, the smoke
check and the benchmark's CPU-baseline leg may import it.  The CUDA library never imports,
links or calls anything here, and nothing here calls the CUDA library.
"""
from .oracle import (  # noqa: F401
    build, lib, splitmix64, fmix64, hash_multiplier, hash_gram, bf16_to_double,
    double_to_bf16, remap, hash_ids, advance_history, gather, gate_conv, forward,
    e4m3_to_double, dequant_e4m3, dequant_table, forward_branches,
)
