"""Offline calibration (Quamba2 method steps 1-3; Quamba-SE write-up 4.1):
the oracle's and the product's host-side implementations are pinned to a
hand-worked case and to numpy, and must agree bit for bit."""
import numpy as np
import pytest

from conftest import golden_rows
from quantized_state_space_b200 import calibrate, synth


def _golden_cluster():
    rows = dict(r.split(":", 1) for r in golden_rows("cluster_case.txt"))
    return (np.array(rows["absmax"].split(), float), int(rows["k"]),
            np.array(rows["cluster_of"].split(), np.int32),
            np.array(rows["scale_numerators"].split(), float))


def test_cluster_golden_oracle(orc):
    a, k, want, num = _golden_cluster()
    cl, sc = orc.cluster_by_absmax(a, k)
    np.testing.assert_array_equal(cl, want)
    np.testing.assert_array_equal(sc, (num / 127.0).astype(np.float32))


def test_cluster_golden_product():
    a, k, want, num = _golden_cluster()
    cl, sc = calibrate.cluster_by_absmax(a, k)
    np.testing.assert_array_equal(cl, want)
    np.testing.assert_array_equal(sc, (num / 127.0).astype(np.float32))


@pytest.mark.parametrize("n,k", [(1536, 8), (80, 8), (77, 5), (10, 10)])
def test_cluster_properties_and_agreement(orc, n, k):
    rng = np.random.default_rng(n + k)
    a = np.abs(rng.standard_normal(n)) * np.exp(rng.uniform(0, 3, n))
    a[rng.choice(n, 3, replace=False)] = a[0]  # ties
    cl, sc = orc.cluster_by_absmax(a, k)
    cp, sp = calibrate.cluster_by_absmax(a, k)
    np.testing.assert_array_equal(cl, cp)
    np.testing.assert_array_equal(sc, sp)
    sizes = np.bincount(cl, minlength=k)
    assert sizes.max() - sizes.min() <= 1 and sizes.sum() == n
    for j in range(k - 1):
        assert a[cl == j].max() <= a[cl == j + 1].min()
    for j in range(k):
        assert sc[j] == np.float32(np.float32(a[cl == j].max()) / np.float32(127)) or \
            sc[j] == np.float32(a[cl == j].max() / 127.0)


def test_channel_absmax_agreement(orc):
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((3, 20, 33)) * 4).astype(np.float16)
    np.testing.assert_array_equal(orc.absmax_per_mid(x, 3, 20, 33), calibrate.channel_absmax(x, 1))
    y = (rng.standard_normal((5, 7, 6, 8))).astype(np.float16)  # (b, L, H, P) heads
    am = orc.absmax_per_mid(y, 35, 6, 8)
    np.testing.assert_array_equal(am, np.abs(y.astype(np.float32)).max(axis=(0, 1, 3)))


@pytest.mark.parametrize("q", [5.0, 99.9, 50.0, 0.0, 100.0])
def test_percentile_matches_numpy(orc, q):
    rng = np.random.default_rng(int(q * 10))
    x = rng.standard_t(3, size=100_001).astype(np.float16)
    got = orc.percentile_abs(x, q)
    ref = np.percentile(np.abs(x.astype(np.float64)), q, method="linear")
    assert abs(got - ref) <= 1e-14 * max(abs(ref), 1e-300)
    assert got == calibrate.percentile_abs(x, q)


def test_softedge_params_agree_with_oracle(orc):
    _, raw = synth.workload_inputs("softedge", batch=1, seqlen=512, dim=64)
    s, lo, hi = calibrate.softedge_params(raw["x"])
    assert lo == np.float32(orc.percentile_abs(raw["x"], 5.0))
    assert hi == np.float32(orc.percentile_abs(raw["x"], 99.9))
    assert s == np.float32(np.float64(hi) / 63.0)
    assert 0 < lo < hi


def test_state_group_scales_agree_with_oracle_absmax(orc):
    rng = np.random.default_rng(5)
    B = rng.standard_normal((2, 3, 16, 40)).astype(np.float16)  # (b, G, N, L)
    gmap = calibrate.state_group_map(3, 16, 4)
    _, sc, _ = orc.quantize_groups(B, 2, 48, 40, gmap, 12, orc.SCALE_ABSMAX)
    np.testing.assert_array_equal(sc, calibrate.state_group_absmax_scales(B, 3, 16, 4, "gnl"))
    B2 = rng.standard_normal((2, 40, 3, 16)).astype(np.float16)  # (b, L, G, N)
    _, sc2, _ = orc.quantize_groups(B2, 80, 48, 1, gmap, 12, orc.SCALE_ABSMAX)
    np.testing.assert_array_equal(sc2, calibrate.state_group_absmax_scales(B2, 3, 16, 4, "lgn"))


def test_ssd_head_clusters():
    rng = np.random.default_rng(9)
    x = (rng.standard_normal((2, 5, 16, 4)) * np.exp(rng.uniform(0, 2, 16))[None, None, :, None])
    x = x.astype(np.float16)
    grp, sc = calibrate.ssd_x_clusters(x, 4)
    assert grp.shape == (64,)
    # every channel of a head shares its cluster
    assert np.all(grp.reshape(16, 4) == grp.reshape(16, 4)[:, :1])


# ---- threshold update (Quamba-SE write-up 4.1), oracle pins ------------------

def test_oracle_softedge_thresholds_alpha_one_equals_host_params(orc):
    """alpha = 1: the thresholds are the percentiles, as the host calibration
    (numpy-pinned percentiles) computes them."""
    rng = np.random.default_rng(41)
    x = (rng.standard_t(3, size=50000)).astype(np.float16)
    s, lo, hi = calibrate.softedge_params(x)
    thr = orc.softedge_thresholds(x, 5.0, 99.9, 1.0, previous=(7.0, 7.0, 7.0))
    assert thr.tolist() == [float(s), float(lo), float(hi)]


def test_oracle_softedge_thresholds_worked_blend(orc):
    """A worked example: every |v| equals 2, so both percentiles are 2; with
    alpha 1/2 and previous (lo, hi) = (4, 6) the blend gives exactly (3, 4) and
    the scale fl32(4 / 63)."""
    x = np.array([2.0, -2.0, 2.0, -2.0], dtype=np.float32)
    thr = orc.softedge_thresholds(x, 5.0, 99.9, 0.5, previous=(0.0, 4.0, 6.0))
    assert thr[1] == 3.0 and thr[2] == 4.0
    assert thr[0] == np.float32(4.0 / 63.0)
    # alpha = 0.1 of the page, previous 0: 0.1 * 2 rounded once to binary32
    thr = orc.softedge_thresholds(x, 5.0, 99.9, float(np.float32(0.1)), previous=(0, 0, 0))
    assert thr[1] == np.float32(float(np.float32(0.1)) * 2.0)


def test_oracle_softedge_thresholds_ignores_nonfinite(orc):
    x = np.array([1.0, np.nan, 3.0, np.inf, -2.0], dtype=np.float32)
    thr = orc.softedge_thresholds(x, 0.0, 100.0, 1.0)
    assert thr[1] == 1.0 and thr[2] == 3.0
