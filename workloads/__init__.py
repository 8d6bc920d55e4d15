"""Workload definitions and seeded input generators shared by the tests, the
benchmark and the CPU oracle's callers.  Holds no step of the method."""
from .configs import Workload, ALL, TINY, AR, CAPACITY, SCALING_32K, LONG, scaling, SCALING_SWEEP  # noqa: F401
from .generate import Inputs, make_inputs, make_keys, make_grad, make_codebooks, make_records, f32_to_bf16_bits, bf16_bits_to_f32  # noqa: F401
