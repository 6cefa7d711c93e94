"""GPU calibration (Quamba2 method steps 1-2: per-channel statistics, sort and
cluster; Quamba-SE write-up 4.1: percentile thresholds with the running
update) against the oracle, bit for bit: the results are exact order
statistics, maxima and one binary32 rounding each."""
import numpy as np
import pytest
import torch

from gpu_util import H, T, status_word
from quantized_state_space_b200 import api, calibrate, synth

pytestmark = pytest.mark.gpu


def _acts(rng, shape, dtype=np.float16, outliers=True):
    x = rng.standard_t(3, size=shape).astype(np.float32)
    if outliers:
        idx = rng.choice(x.size, size=max(1, x.size // 2000), replace=False)
        x.reshape(-1)[idx] *= rng.uniform(100, 1000, size=idx.size)
    return x.astype(dtype)


@pytest.mark.parametrize("layout", ["rows", "cols", "general", "f32"])
def test_group_absmax_vs_oracle(orc, layout):
    rng = np.random.default_rng({"rows": 1, "cols": 2, "general": 3, "f32": 4}[layout])
    if layout == "rows":       # Mamba-1 x (b, d, L): channel rows
        outer, mid, inner = 3, 96, 640
    elif layout == "cols":     # Mamba-2 x (b L, H P): channel columns
        outer, mid, inner = 700, 320, 1
    elif layout == "general":  # inner not a multiple of 16
        outer, mid, inner = 5, 24, 37
    else:
        outer, mid, inner = 2, 64, 512
    x = _acts(rng, (outer, mid, inner), np.float32 if layout == "f32" else np.float16)
    x.reshape(-1)[rng.choice(x.size, size=4, replace=False)] = [np.nan, np.inf, -np.inf, np.nan]
    st = status_word()
    got = api.group_absmax(T(x), outer, mid, inner, T(np.arange(mid, dtype=np.int32)), mid,
                           status=st)
    ref = orc.absmax_per_mid(x, outer, mid, inner)
    np.testing.assert_array_equal(H(got), ref.astype(np.float32))
    assert int(H(st)[0]) & 1  # the non-finite elements were seen


@pytest.mark.parametrize("n,k", [(1536, 8), (5120, 8), (7, 7), (1000, 1), (65536, 13), (33, 5)])
def test_cluster_by_absmax_vs_oracle(orc, n, k):
    rng = np.random.default_rng(n + k)
    a = rng.uniform(0, 10, size=n).astype(np.float32)
    a[rng.choice(n, size=n // 4, replace=False)] = a[0]  # many ties: index order decides
    a[1] = 0.0
    cl, sc = api.cluster_by_absmax(T(a), k)
    rc, rs = orc.cluster_by_absmax(a.astype(np.float64), k)
    np.testing.assert_array_equal(H(cl), rc)
    np.testing.assert_array_equal(H(sc), rs)


def test_cluster_map_on_device_equals_host_calibration():
    """The offline step a0 on the device (channel maxima, then sort and
    cluster) gives the host calibration's cluster map and scales."""
    dm, raw = synth.workload_inputs("tiny")
    x = raw["x"]
    b, d, L = x.shape
    amax = api.group_absmax(T(x), b, d, L, T(np.arange(d, dtype=np.int32)), d)
    cl, sc = api.cluster_by_absmax(amax, 4)
    hc, hs = calibrate.m1_x_clusters(x, 4)
    np.testing.assert_array_equal(H(cl), hc)
    np.testing.assert_array_equal(H(sc), hs)


@pytest.mark.parametrize("dtype,n", [(np.float16, 1000), (np.float16, 3_000_001),
                                     (np.float32, 4099), (np.float32, 2_000_003)])
def test_percentile_abs_vs_oracle(orc, dtype, n):
    rng = np.random.default_rng(n)
    x = _acts(rng, (n,), dtype)
    x[rng.choice(n, size=3, replace=False)] = [np.nan, np.inf, -0.0]
    qs = [0.0, 5.0, 99.9, 100.0]
    got = H(api.percentile_abs(T(x), qs))
    ref = np.array([orc.percentile_abs(x, q) for q in qs], dtype=np.float32)
    np.testing.assert_array_equal(got, ref)
    got = H(api.percentile_abs(T(x), [50.0, 37.5]))
    ref = np.array([orc.percentile_abs(x, q) for q in (50.0, 37.5)], dtype=np.float32)
    np.testing.assert_array_equal(got, ref)


def test_percentile_abs_edge_cases(orc):
    empty = np.zeros(0, np.float32)
    assert H(api.percentile_abs(T(np.ones(4, np.float32))[:0], [50.0]))[0] == 0.0
    allnan = np.full(17, np.nan, np.float32)
    assert H(api.percentile_abs(T(allnan), [5.0]))[0] == orc.percentile_abs(allnan, 5.0) == 0.0
    one = np.array([-3.5], np.float16)
    assert H(api.percentile_abs(T(one), [0.0, 99.9]))[1] == 3.5
    del empty


@pytest.mark.parametrize("dtype", [np.float16, np.float32])
def test_softedge_calibrate_vs_oracle(orc, dtype):
    rng = np.random.default_rng(77)
    x = _acts(rng, (1_234_567,), dtype)
    thr = api.softedge_calibrate(T(x))
    s, lo, hi = calibrate.softedge_params(x)
    assert H(thr).tolist() == [float(s), float(lo), float(hi)]
    # running update with the page's alpha on a second batch
    x2 = _acts(rng, (777_777,), dtype)
    prev = H(thr).copy()
    alpha = float(np.float32(0.1))
    api.softedge_calibrate(T(x2), thr, alpha=alpha)
    ref = orc.softedge_thresholds(x2, 5.0, 99.9, alpha, previous=tuple(prev))
    np.testing.assert_array_equal(H(thr), ref)
