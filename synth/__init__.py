"""Seeded synthetic inputs for the n-gram embedding lookup.

This package generates inputs only: token-id streams, the vocabulary-compression table,
and counter-based bf16 fills for tables, weights, hidden states and decode state (and e4m3
codes for FP8 tables).  It
holds none of the lookup's arithmetic (no hashing of grams, no gathering, no gating), so
both the CPU oracle and the CUDA path can be fed from it without sharing method code.

Every generator is a pure function of (seed, tensor id, element counter): any element of
any tensor, including rows of a 95 GiB table, can be regenerated on the CPU without
materialising the tensor, and the GPU fill kernel produces bit-identical values.
"""
from .fill import (FillSpec, fill_bf16, fill_rows_bf16, bf16_to_float, float_to_bf16_rne, fill_fp8,
                   fill_rows_fp8, encode_e4m3_int, fp8_scale_for_sigma)
from .streams import zipf_ids, uniform_ids, remap_table, phrase_stream
from .workloads import Workload, WORKLOADS, get_workload, largest_prime_below

__all__ = [
    "FillSpec", "fill_bf16", "fill_rows_bf16", "bf16_to_float", "float_to_bf16_rne", "fill_fp8",
    "fill_rows_fp8", "encode_e4m3_int", "fp8_scale_for_sigma",
    "zipf_ids", "uniform_ids", "remap_table", "phrase_stream",
    "Workload", "WORKLOADS", "get_workload", "largest_prime_below",
]
