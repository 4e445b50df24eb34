"""Shared helpers of the GPU parity tests: seeded inputs on the device and the
comparison rules (the oracle is the reference; only tests call it)."""
from __future__ import annotations

import numpy as np
import torch

from diffusion_transformer_video_b200 import workloads as wl

# Tolerances of the stated accuracy targets: attention max abs 2e-2 / mean abs 2e-3 on unit-normal inputs;
# modulation kernels 1e-2 max abs, measured as |gpu - ref| <= 1e-2 + half a bf16 ulp of ref
# (a correctly rounded bf16 output of |ref| >= 4 is already 1/64 away from ref).
ATTN_MAX, ATTN_MEAN = 2e-2, 2e-3
MOD_ABS = 1e-2


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> contiguous bf16 CUDA tensor (same bits)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def from_dev(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def f64(bits: np.ndarray) -> np.ndarray:
    return wl.bf16_bits_to_f64(bits)


def half_ulp_bf16(ref: np.ndarray) -> np.ndarray:
    a = np.abs(ref)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 8).astype(np.int64))


def check_modulation(gpu: np.ndarray, ref: np.ndarray, what: str) -> dict:
    err = np.abs(gpu - ref)
    bound = MOD_ABS + half_ulp_bf16(ref)
    bad = err > bound
    info = {"max_abs": float(err.max()), "mean_abs": float(err.mean()),
            "violations": int(bad.sum())}
    assert not bad.any(), f"{what}: {info}"
    return info


def check_attention(gpu: np.ndarray, ref: np.ndarray, what: str) -> dict:
    err = np.abs(gpu - ref)
    info = {"max_abs": float(err.max()), "mean_abs": float(err.mean())}
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    assert info["max_abs"] <= ATTN_MAX and info["mean_abs"] <= ATTN_MEAN, f"{what}: {info}"
    return info
