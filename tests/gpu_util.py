"""Helpers for the GPU parity tests: move bfloat16 bit patterns to and from the
device and compare a GPU result with the float64 oracle.

Parity bar for bfloat16 outputs: max-abs error <= 2e-2 and relative L2 error
||gpu - oracle||_2 / ||oracle||_2 <= 5e-3 over the compared elements, against
the unrounded oracle.  float32 softmax weights: every row sums to 1 within
1e-5 and blocked keys are exactly 0.
"""
import numpy as np
import torch

MAX_ABS = 2e-2
REL_L2 = 5e-3
ROW_SUM = 1e-5


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return (bits(t).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return t.detach().cpu().double().numpy()


def errors(gpu, ref):
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), "non-finite GPU output"
    d = g - r
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(r), 1e-300))
    return max_abs, rel


def assert_parity(gpu, ref, what="", max_abs=MAX_ABS, rel_l2=REL_L2):
    ma, rl = errors(gpu, ref)
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max-abs {ma:.3e} (bar {max_abs}), rel-L2 {rl:.3e} (bar {rel_l2})"
    return ma, rl
