"""Shared test utilities: device upload of seeded inputs and tolerance checks."""
import numpy as np
import torch

import synth


def to_device(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Upload float32 values that sit on the dtype grid (exactly, via bit patterns for bf16)."""
    if dtype == "bf16":
        bits = synth.bf16_bits_from_f32(np.ascontiguousarray(x, np.float32))
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()


def to_numpy(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_fro(got: np.ndarray, want: np.ndarray) -> float:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    den = np.linalg.norm(want)
    num = np.linalg.norm(got - want)
    return float(num / den) if den > 0 else float(num)


def torch_dtype(dtype: str):
    return torch.bfloat16 if dtype == "bf16" else torch.float32
