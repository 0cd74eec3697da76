"""Helpers for the GPU tests: move seeded inputs to the device, read results
back, and the parity metrics (max-abs and relative L2 against the oracle)."""
import numpy as np
import torch

from causal_attention_rtr_b200 import synth

# Attention tolerance for bf16 storage against the fp64 oracle on identical
# input bits: max |gpu - oracle| <= 2e-2 and ||gpu - oracle||_2 / ||oracle||_2
# <= 5e-3.
MAX_ABS = 2e-2
REL_L2 = 5e-3


def dev(a: np.ndarray) -> torch.Tensor:
    """Device tensor holding exactly the bits of ``a`` (uint16 bf16 patterns
    become a bfloat16 tensor; float32 stays float32)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).cuda()
    if a.dtype == np.float32:
        return torch.from_numpy(a.copy()).cuda()
    raise TypeError(a.dtype)


def host_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bits of a device tensor (uint16 for bf16, float32 otherwise)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def host_f64(t: torch.Tensor) -> np.ndarray:
    b = host_bits(t)
    if b.dtype == np.uint16:
        return synth.bf16_bits_to_f32(b).astype(np.float64)
    return b.astype(np.float64)


def empty_like_raw(shape, dtype: str) -> torch.Tensor:
    return torch.empty(shape, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device="cuda")


def errors(got: np.ndarray, want: np.ndarray):
    diff = got - want
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    denom = float(np.linalg.norm(want.ravel()))
    rel = float(np.linalg.norm(diff.ravel()) / denom) if denom > 0 else float(np.linalg.norm(diff.ravel()))
    return max_abs, rel


def assert_close(got, want, what=""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    max_abs, rel = errors(got, want)
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel
