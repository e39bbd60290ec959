"""Helpers shared by the GPU parity tests: device transfer of the seeded inputs and the
error metric. Nothing here computes any step of the method."""
import numpy as np
import torch

import tg_inputs as ti

# tolerances of the gated-prefill path: max-abs-relative error per tensor
TOL = {"f32": 1e-4, "bf16": 2e-2}


def max_abs_rel(x, r) -> float:
    """max |x - r| / max |r| over the tensor (0 for empty tensors)."""
    x = np.asarray(x, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    if r.size == 0:
        return 0.0
    return float(np.max(np.abs(x - r)) / max(float(np.max(np.abs(r))), 1e-30))


def to_dev(a, dtype: str, device="cuda"):
    """Stored array (float32, or bf16 bits as uint16) -> torch tensor on the GPU, same bytes."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(device)


def from_dev(t) -> np.ndarray:
    """torch tensor -> float64 numpy (bf16 widened exactly)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.numpy().astype(np.float64)


def bits(t) -> np.ndarray:
    """Raw bits of a tensor for bit-exact comparisons."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy()
    return t.numpy()


def widen(a, dtype):
    return ti.widen(a, dtype)
