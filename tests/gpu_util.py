"""Helpers shared by the GPU parity tests (oracle on host copies of the
same seeded inputs the CUDA path consumed)."""

from __future__ import annotations

import numpy as np
import torch

import oracle as O


def host_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 host copy of a bf16/fp32 device tensor."""
    return t.detach().to("cpu").double().numpy()


def host_dequant(codes: torch.Tensor, scale: torch.Tensor, group_dims: int) -> np.ndarray:
    """Dequantised float64 value of FP8 e4m3 codes with per-token scales,
    using the oracle's own e4m3 decoder."""
    c = codes.detach().to("cpu").view(torch.uint8).numpy()
    return O.dequantize(c, scale.detach().to("cpu").numpy(), group_dims)


def indexer_host_inputs(d: dict):
    """(q, k, w) as float64 host arrays for the oracle."""
    if "q_scale" in d:
        q = host_dequant(d["qI"], d["q_scale"], 2)
        k = host_dequant(d["kI"], d["k_scale"], 1)
    else:
        q = host_f64(d["qI"])
        k = host_f64(d["kI"])
    return q, k, host_f64(d["w"])
