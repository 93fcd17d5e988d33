"""Helpers shared by the GPU tests: moving generator arrays onto the device
and reading results back exactly, plus the stated tolerances."""

import numpy as np
import pytest
import torch

from _pins import rel_err as _rel_err

# Absolute floor of the error denominator: results whose exact value is 0
# (e.g. gk of a one-token sequence) are compared against 1e-6 instead of the
# oracle's round-off.
ABS_FLOOR = 1e-6


def rel_err(x, ref):
    """max_i |x_i - ref_i| / max(|ref_i|, rms(ref), 1e-6)."""
    return _rel_err(x, ref, floor=ABS_FLOOR)

# Max relative error (elementwise, denominator floored at the reference RMS)
# allowed against the fp64 oracle: 1e-4 for float32 I/O, 2e-2 for bf16 I/O
# with float32 state.
TOL = {"f32": 1e-4, "bf16": 2e-2}


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def dev(a: np.ndarray) -> torch.Tensor:
    """float32 arrays -> float32 tensor; uint16 arrays (bf16 bits) -> bf16 tensor."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    if a.dtype == np.int32:
        return torch.from_numpy(a).cuda()
    return torch.from_numpy(a.astype(np.float32, copy=False)).cuda()


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_no_device_error():
    from rwkv_wkv_linear_mix_b200 import wkv
    assert wkv.device_error(reset=True) == 0
