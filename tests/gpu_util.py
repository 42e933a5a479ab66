"""Shared helpers of the GPU parity tests (inputs from the workload module,
oracle calls, comparison metrics)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from bit_quantized_flashattention_smooth_b200 import workloads as W

# Output tolerance: |dO| <= 1e-2 * max|O| + 1e-3 elementwise and cosine >= 0.9999
# (the stated bar for floating-point outputs against the oracle).
ATOL_REL, ATOL_ABS, COS_MIN = 1e-2, 1e-3, 0.9999


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def compare_out(gpu: np.ndarray, ref: np.ndarray):
    """Returns (ok, max_err, bound, cosine)."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    bound = ATOL_REL * np.max(np.abs(ref)) + ATOL_ABS
    err = float(np.max(np.abs(gpu - ref)))
    cos = float(np.sum(gpu * ref) / (np.linalg.norm(gpu) * np.linalg.norm(ref) + 1e-300))
    return (err <= bound and cos >= COS_MIN), err, bound, cos


def oracle_quantize(q, k, v, s, inv_s, fmt):
    """Oracle quantization of CPU torch tensors; returns plain-layout dict and
    the tiled scale bytes."""
    qz = oracle.quantize_qkv(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                             None if s is None else s, None if inv_s is None else inv_s, fmt)
    return qz, oracle.tile_scales(qz)


def synthetic(B, Hq, Hkv, N, d, seed, dtype=torch.bfloat16, outlier=8.0):
    """Small seeded inputs with a few outlier K channels (for ragged shapes)."""
    g = np.random.Generator(np.random.PCG64(seed))
    q = g.standard_normal((B, Hq, N, d), dtype=np.float32)
    k = g.standard_normal((B, Hkv, N, d), dtype=np.float32)
    v = g.standard_normal((B, Hkv, N, d), dtype=np.float32)
    if outlier:
        k[..., -3:] = outlier * np.abs(k[..., -3:])
    return (torch.from_numpy(q).to(dtype), torch.from_numpy(k).to(dtype), torch.from_numpy(v).to(dtype))
