"""Seeded synthetic workloads shared by the tests, the benchmark and the oracle's callers.

This package generates inputs only.  It holds none of the attention method's arithmetic
(no quantisation, routing, scores or softmax), so both the CUDA path and the CPU oracle can
take their inputs from it without sharing any of the method's code.
"""
from .gen import (CONFIGS, Tensors, Workload, config_by_name, make_workload,  # noqa: F401
                  sample_rows, sample_tiles, to_16bit, bf16_bits_to_f32)
