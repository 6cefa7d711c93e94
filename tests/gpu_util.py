"""Helpers of the GPU parity tests."""
import numpy as np
import pytest
import torch

# tolerances stated by the method's target: max |y - y_ref| <= 2e-3 max |y_ref|
# and final-state relative L2 <= 1e-4
Y_TOL = 2e-3
STATE_TOL = 1e-4


def dev():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    return torch.device("cuda:0")


def T(a, dtype=None):
    """numpy -> contiguous CUDA tensor (float16 stays float16)."""
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.to(dev())


def H(t):
    return t.detach().cpu().numpy()


def y_err(y_gpu, y_ref):
    y = np.asarray(y_gpu, np.float64)
    r = np.asarray(y_ref, np.float64)
    return float(np.max(np.abs(y - r)) / max(np.max(np.abs(r)), 1e-30))


def state_err(h_gpu, h_ref):
    h = np.asarray(h_gpu, np.float64)
    r = np.asarray(h_ref, np.float64)
    return float(np.linalg.norm(h - r) / max(np.linalg.norm(r), 1e-30))


def assert_scan_close(y_gpu, y_ref, h_gpu=None, h_ref=None):
    e = y_err(y_gpu, y_ref)
    assert e <= Y_TOL, "y error %.3g > %.1g" % (e, Y_TOL)
    if h_gpu is not None:
        s = state_err(h_gpu, h_ref)
        assert s <= STATE_TOL, "state rel-L2 %.3g > %.1g" % (s, STATE_TOL)
    return e


def status_word():
    return torch.zeros(1, dtype=torch.int32, device=dev())
