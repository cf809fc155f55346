"""Shared test helpers: host<->device marshalling of generated inputs and the
parity metrics.  No method arithmetic lives here."""
import numpy as np
import torch

import svg_inputs as si

# Output tolerance for floating-point parity (bf16 kernels against the float64
# oracle): max-abs error 2e-2 and relative RMS ||o - o_ref||_2 / ||o_ref||_2
# 1e-2.  A bf16 output cannot be closer to the float64 value than half a bf16
# ulp, which exceeds 2e-2 once |o_ref| >= 8 (ulp 0.0625); there a value next
# to a rounding midpoint may round either way.  The per-element max-abs bound
# is therefore max(2e-2, half a bf16 ulp at |o_ref| + 1e-3): 2e-2 wherever
# bf16 can meet it, and otherwise the representation step plus 1e-3 of
# arithmetic error.
MAX_ABS = 2e-2
REL_RMS = 1e-2
# relative margin below which a profiling choice is not compared
MODE_MARGIN = 1e-3


def to_device(x: np.ndarray, device="cuda") -> torch.Tensor:
    """Generated tensor (uint16 bf16 bits or float32) -> torch on device."""
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).to(device)


def to_float64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw element bits (for bit-exact comparison)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy()
    return t.numpy()


def half_ulp_bf16(ref: np.ndarray) -> np.ndarray:
    a = np.abs(ref)
    e = np.floor(np.log2(np.maximum(a, 1e-30)))
    return np.where(a > 0, 2.0 ** (e - 8), 0.0)


def assert_close(got: np.ndarray, ref: np.ndarray, what: str = "", bf16: bool = True):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    bound = np.maximum(MAX_ABS, half_ulp_bf16(ref) + 1e-3) if bf16 else MAX_ABS
    worst = np.unravel_index(np.argmax(err - bound), err.shape) if err.size else ()
    assert (err <= bound).all(), (
        f"{what}: max-abs {err.max():.4g} at {worst} (ref {ref[worst]:.5g}, got {got[worst]:.5g})")
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(got - ref) / nref if nref > 0 else np.linalg.norm(got)
    assert rel <= REL_RMS, f"{what}: rel-RMS {rel:.4g}"
    return float(err.max()), float(rel)


def workload_tensors(wl, seed=None, types_seed=None, device="cuda"):
    q, k, v, types = si.generate(wl, seed=seed, types_seed=types_seed)
    return (q, k, v), tuple(to_device(x, device) for x in (q, k, v)), types
