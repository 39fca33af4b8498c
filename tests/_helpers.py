"""Shared test plumbing: conversions between torch tensors and the oracle's
fp64 arrays. No arithmetic of the head lives here."""
import numpy as np
import torch


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact fp64 copy of a CPU or CUDA tensor (bf16 and fp32 convert exactly)."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def dtype_name(t: torch.dtype) -> str:
    return {torch.bfloat16: "bf16", torch.float32: "fp32"}[t]


def to_dev(d: dict, device="cuda") -> dict:
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
