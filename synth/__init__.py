"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

Holds no optimizer or planner arithmetic: tensor shape lists for the bucket
workloads and a counter-based random generator (SplitMix64 + Box-Muller, in
``gen.c``).  Every array handed to either side comes from here, so both see
the same bytes.
"""
from .workloads import (  # noqa: F401
    HPARAMS,
    TensorSpec,
    Workload,
    workload,
    WORKLOAD_NAMES,
    ragged_mix,
)
from .rng import (  # noqa: F401
    build,
    stream_key,
    normal_f32,
    normal_bf16,
    uniform_f64,
    load_lib,
)
