"""Helpers for the GPU tests: move bf16 bit patterns to the device and back.

No arithmetic of the method lives here.
"""

import numpy as np

# Tolerance of the path for bf16 outputs against the float64 oracle.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def dev_bf16(bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def dev(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_f64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def host_bits(t) -> np.ndarray:
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def assert_close_bf16(got: np.ndarray, want: np.ndarray, what: str,
                      max_abs: float = MAX_ABS, mean_abs: float = MEAN_ABS) -> None:
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - want)
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert mx <= max_abs and mean <= mean_abs, f"{what}: max|d|={mx:.3g} mean|d|={mean:.3g}"
