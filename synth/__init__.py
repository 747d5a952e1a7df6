"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This package holds no arithmetic of the quantized linear layer itself: it only
draws random bf16 tensors with the shapes and value distributions of the FLUX
DiT linear layers, and names the workloads.  Both the CUDA path and the CPU
oracle are fed from here, so that they see identical input bits.
"""
from .tensors import bf16_bits_from_f64, bf16_bits_to_f32, draw, rng_for  # noqa: F401
from .workloads import WORKLOADS, Workload, make_inputs  # noqa: F401
