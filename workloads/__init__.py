"""Seeded synthetic workloads shared by the tests, the benchmark and the oracle."""
from .synthetic import (Workload, make_workload, make_chunked_workload, make_config, ragged_lengths,
                        quantize_e4m3, page_kv, CONFIG_NAMES)
from .long_context import make_long_device_inputs

__all__ = ["Workload", "make_workload", "make_chunked_workload", "make_config", "ragged_lengths", "quantize_e4m3",
           "page_kv", "CONFIG_NAMES", "make_long_device_inputs"]
