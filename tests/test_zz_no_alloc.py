"""Allocation-free percentile entry points (the library's static device
scratch instead of a caller workspace): the same bytes as the workspace
calls, no device allocation, and the oversize rule is stated by the size
query.  Collected last."""
import ctypes as C

import numpy as np
import pytest
import torch

from gpu_util import H, T
from quantized_state_space_b200 import _native as N
from quantized_state_space_b200 import api


def test_noalloc_symbols_exported():
    L = N.lib()
    assert hasattr(L, "ssmq_percentile_abs_noalloc")
    assert hasattr(L, "ssmq_softedge_calibrate_noalloc")


def test_noalloc_validation_before_launch():
    """Argument errors come back before any device call (no GPU needed)."""
    L = N.lib()
    q = (C.c_double * 2)(50.0, 120.0)
    fake = 1 << 20
    assert L.ssmq_percentile_abs_noalloc(None, N.F16, 16, q, 1, fake, None) == N.ERR_INVALID_ARG
    assert L.ssmq_percentile_abs_noalloc(fake, N.F16, 16, q, 2, fake, None) == N.ERR_INVALID_ARG
    assert L.ssmq_percentile_abs_noalloc(fake, N.F16, 16, q, 5, fake, None) == N.ERR_INVALID_ARG
    assert L.ssmq_softedge_calibrate_noalloc(fake, N.F32, 16, 5.0, 99.9, 0.0, fake,
                                             None) == N.ERR_INVALID_ARG
    assert L.ssmq_softedge_calibrate_noalloc(fake, N.F32, 16, 99.9, 5.0, 1.0, fake,
                                             None) == N.ERR_INVALID_ARG


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [np.float16, np.float32])
def test_noalloc_equals_workspace_calls(dtype):
    rng = np.random.default_rng(5)
    x = (rng.standard_t(3, size=999_999) * rng.choice([1.0, 300.0], size=999_999,
                                                      p=[0.999, 0.001])).astype(dtype)
    xt = T(x)
    qs = [5.0, 50.0, 99.9, 100.0]
    ref = H(api.percentile_abs(xt, qs))
    out = torch.empty(len(qs), dtype=torch.float32, device=xt.device)
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated()
    N.ssmq_percentile_abs_noalloc(xt, xt.numel(), qs, out)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before
    np.testing.assert_array_equal(H(out), ref)
    thr_ws = api.softedge_calibrate(xt)
    thr = torch.zeros(3, dtype=torch.float32, device=xt.device)
    N.ssmq_softedge_calibrate_noalloc(xt, xt.numel(), 5.0, 99.9, 1.0, thr)
    np.testing.assert_array_equal(H(thr), H(thr_ws))
    # the running update on the static scratch, twice in a row on one stream
    prev = H(thr).copy()
    N.ssmq_softedge_calibrate_noalloc(xt[: 500_000], 500_000, 5.0, 99.9, 0.1, thr)
    thr2 = T(prev)
    api.softedge_calibrate(xt[: 500_000], thr2, alpha=0.1)
    np.testing.assert_array_equal(H(thr), H(thr2))
