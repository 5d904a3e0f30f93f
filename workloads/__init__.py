"""Seeded synthetic inputs for the paged decode path.

This package only draws numbers and lays them out (context lengths, a shuffled
physical block pool, block tables, slot mappings, copy-on-write pairs, q/K/V
values rounded to 16-bit floats). It computes none of the attention arithmetic,
so both the CPU oracle and the CUDA library can be fed from it without sharing
any of the method's code.
"""
from .gen import (  # noqa: F401
    DecodeCase,
    CONFIGS,
    make_case,
    make_config,
    round_to_bits,
    bits_to_f32,
    NAN_BITS,
    PrefillCase,
    PREFILL_CONFIGS,
    make_prefill_case,
    make_prefill_config,
)
