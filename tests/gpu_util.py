"""Helpers shared by the GPU parity tests (no arithmetic of the method here)."""
import numpy as np
import torch

from block_attention_b200 import synth


def to_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    if a.dtype == np.uint16:  # bf16 bit patterns
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def to_host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return synth.bf16_to_f32(t.view(torch.int16).numpy().view(np.uint16))
    return t.numpy()


def rel_err_rows(got: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Per (b, row, head): max |got - ref| / max(max |ref|, 1e-6) over the head dim."""
    got = np.asarray(got, np.float64)
    num = np.abs(got - ref).max(axis=-1)
    den = np.maximum(np.abs(ref).max(axis=-1), 1e-6)
    return num / den


TOL = {"f32": 1e-5, "bf16": 2e-2}
