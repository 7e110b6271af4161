"""Seeded synthetic inputs shared by the fp64 oracle and the CUDA path.

This package only draws numbers and lays out shapes. It holds none of the
method's arithmetic (no layer, no attention, no modulation, no Euler step):
both the oracle and the CUDA path receive its arrays as plain inputs.
"""
from .gen import (  # noqa: F401
    GOLDEN_GAMMA,
    splitmix64_mix,
    stream_key,
    uniform_u64,
    uniform01,
    normal,
    normal_torch,
)
from .configs import (  # noqa: F401
    ModelShape,
    Workload,
    WORKLOADS,
    make_workload,
)
