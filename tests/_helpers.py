"""Shared helpers for the GPU parity tests: moving seeded bf16 inputs to the
device and reading results back. No attention arithmetic here."""

import numpy as np
import torch

from synthetic import attention_inputs, bf16_bits_to_f32

# Tolerances of the workload statement (bf16 path vs the fp64 oracle run on
# the bf16-rounded inputs).
O_MAX_ABS = 2e-2
LSE_MAX_ABS = 1e-3
GRAD_REL_L2 = 1e-2


def to_device_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def make_inputs(B, Hq, Hkv, N, d, seed, outlier_rate=0.0, with_dout=True):
    bits = attention_inputs(B, Hq, Hkv, N, d, seed, outlier_rate=outlier_rate, with_dout=with_dout)
    dev = {n: to_device_bf16(a) for n, a in bits.items()}
    host = {n: bf16_bits_to_f32(a).astype(np.float64) for n, a in bits.items()}
    return dev, host


# Relative L2 is undefined when the exact gradient is zero (N = 1: one key,
# so dS = P (dP - D) = 0 and dQ = dK = 0 exactly). The denominator is floored
# at an RMS of 1e-3 per element, far below the O(0.1..1) gradients of the
# N(0,1) workloads, so the floor only matters for all-zero references.
GRAD_RMS_FLOOR = 1e-3


def rel_l2(a, b):
    floor = GRAD_RMS_FLOOR * np.sqrt(b.size)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), floor))
