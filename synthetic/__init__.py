"""Seeded synthetic inputs shared by the oracle tests and the CUDA path.

This package draws random numbers and names workload shapes. It holds none of
the attention arithmetic: no products, no softmax, no quantisation.
"""

from .gen import (  # noqa: F401
    splitmix64,
    uniform01,
    normal,
    bf16_round,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    sign_vector,
    attention_inputs,
    STREAM_Q,
    STREAM_K,
    STREAM_V,
    STREAM_DO,
    STREAM_OUTLIER,
    STREAM_SIGN,
)
from .configs import WORKLOADS, Workload  # noqa: F401
