"""Seeded synthetic inputs shared by tests, the benchmark and the oracle (no method arithmetic)."""
from .synth import (DTYPE_NAMES, FULL_CONFIGS, SMALL_CONFIGS, Workload, decode_workload,  # noqa: F401
                    lognormal_lengths, make, mixed_workload, shared_prefix_workload,
                    to_numpy_raw, torch_dtype, values)
