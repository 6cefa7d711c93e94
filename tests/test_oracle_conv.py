"""Pins of the oracle's producer step: the causal depthwise convolution and
SiLU that form the Mamba-1 scan input, evaluated in binary32 so that the
quantizer's code is decided on the same value by the oracle and the kernel.

Each step is pinned to something other than itself: the exponential and
SiLU to double-precision mathematics (numpy) within stated ulp bounds over a
dense sweep of binary32 inputs; the convolution to hand-worked values
(tests/golden/conv_case.txt) and to an independent double-precision
convolution; the carried conv state to the unsplit call."""
import numpy as np
import pytest

from conftest import golden_rows


def _ulp(ref32):
    return np.spacing(np.abs(ref32).astype(np.float32)).astype(np.float64)


def _fp32_sweep(lo, hi, stride):
    """Every stride-th binary32 value in [lo, hi] (both signs by bit pattern)."""
    pos = np.arange(0, np.float32(max(hi, 0)).view(np.uint32) + 1, stride, dtype=np.uint64)
    neg = np.arange(0, np.float32(max(-lo, 0)).view(np.uint32) + 1, stride, dtype=np.uint64)
    v = np.concatenate([pos.astype(np.uint32).view(np.float32),
                        -(neg.astype(np.uint32).view(np.float32))])
    return v[(v >= lo) & (v <= hi)]


def test_exp_f32_within_two_ulp(orc):
    """e^v over every 61st binary32 value in [-87, 88] (about 35 M inputs):
    within 2 ulp of the correctly rounded double-precision e^v."""
    v = _fp32_sweep(-87.0, 88.0, 61)
    assert v.size > 30_000_000
    got = orc.exp_f32(v).astype(np.float64)
    ref = np.exp(v.astype(np.float64))
    err = np.abs(got - ref) / _ulp(ref.astype(np.float32))
    assert err.max() <= 2.0, "exp_f32 max error %.3f ulp at v=%r" % (err.max(), v[err.argmax()])
    # range ends of the definition and exact points
    e = orc.exp_f32(np.array([0.0, 88.5, 1e30, -87.5, -1e30, np.inf, -np.inf, np.nan],
                             np.float32))
    assert e[0] == 1.0 and np.isinf(e[1]) and np.isinf(e[2]) and np.isinf(e[5])
    assert e[3] == 0.0 and e[4] == 0.0 and e[6] == 0.0 and np.isnan(e[7])


def test_exp_f32_integer_points(orc):
    """e^k for integers k: the reduction leaves r = k (1 - ln2 ratio) tiny or
    exact; compare with the double value (1 ulp)."""
    k = np.arange(-87, 89, dtype=np.float32)
    got = orc.exp_f32(k).astype(np.float64)
    ref = np.exp(k.astype(np.float64))
    assert (np.abs(got - ref) / _ulp(ref.astype(np.float32))).max() <= 1.0


def test_silu_f32_bound(orc):
    """silu(a) = a / (1 + e^-a) over every 53rd binary32 value in [-86, 90]:
    within 4 ulp of the double-precision value (the exponential's 2 ulp, the
    rounding of 1 + e, of the reciprocal and of the product); below -86 the
    definition may give -0 where the value is below 1e-35 in magnitude."""
    a = _fp32_sweep(-86.0, 90.0, 53)
    got = orc.silu_f32(a).astype(np.float64)
    ad = a.astype(np.float64)
    ref = ad / (1.0 + np.exp(-ad))
    big = np.abs(ref) > 1e-30
    err = np.abs(got - ref)[big] / _ulp(ref[big].astype(np.float32))
    assert err.max() <= 4.0, "silu_f32 max error %.3f ulp" % err.max()
    assert np.all(np.abs(got[~big] - ref[~big]) <= 1e-30)
    s = orc.silu_f32(np.array([0.0, -0.0, -100.0, 100.0, np.inf, np.nan], np.float32))
    assert s[0] == 0.0 and s[2] == 0.0 and s[3] == 100.0 and np.isinf(s[4]) and np.isnan(s[5])


def test_conv_golden(orc):
    """The hand-worked convolution (golden file): the oracle's u equals silu of
    the hand values (exact in binary32) within the SiLU bound."""
    rows = [r.split() for r in golden_rows("conv_case.txt")]
    x = np.array([[[1, 2, 0.5, -1, 4]]], np.float16)
    w = np.array([[0.25, 0.5, -1.0, 2.0]], np.float32)
    bias = np.array([0.125], np.float32)
    prev = np.array([[[3, -2, 0.5]]], np.float16)
    u0, st0, _ = orc.conv_silu(x, w, bias)
    u1, st1, _ = orc.conv_silu(x, w, bias, x_prev=prev)
    for state, t, a in rows:
        u = (u0 if state == "none" else u1)[0, 0, int(t)]
        a = float(a)
        ref = a / (1.0 + np.exp(-a))
        assert abs(u - ref) <= 4 * np.spacing(np.float32(abs(ref))), (state, t, u, ref)
    np.testing.assert_array_equal(st0[0, 0], np.array([0.5, -1, 4], np.float16))
    np.testing.assert_array_equal(st1, st0)


def _conv_ref(x, w, bias, prev):
    """Independent double-precision reference: numpy correlation over the
    state-padded rows, then silu in double; also the bound of the binary32
    chain's rounding (sum of |terms| times a few units of 2^-24)."""
    b, d, L = x.shape
    W = w.shape[1]
    pad = np.zeros((b, d, W - 1)) if prev is None else prev.astype(np.float64)
    full = np.concatenate([pad, x.astype(np.float64)], axis=-1)
    a = np.zeros((b, d, L)) + (0.0 if bias is None else bias.astype(np.float64)[None, :, None])
    mag = np.abs(a).copy()
    for k in range(W):
        term = w[None, :, k, None].astype(np.float64) * full[..., k:k + L]
        a += term
        mag += np.abs(term)
    return a / (1.0 + np.exp(-a)), mag


@pytest.mark.parametrize("W,with_bias,with_prev", [(4, True, False), (4, True, True),
                                                   (3, False, True), (2, True, True),
                                                   (1, True, False), (4, False, False)])
def test_conv_silu_vs_double(orc, W, with_bias, with_prev):
    rng = np.random.default_rng(100 + 10 * W + 2 * with_bias + with_prev)
    b, d, L = 2, 7, 53
    x = (rng.standard_normal((b, d, L)) * rng.choice([0.5, 3.0], size=(b, d, 1))).astype(np.float16)
    w = (rng.standard_normal((d, W)) * 0.5).astype(np.float32)
    bias = (rng.standard_normal(d) * 0.3).astype(np.float32) if with_bias else None
    prev = rng.standard_normal((b, d, W - 1)).astype(np.float16) if with_prev else None
    u, st, nonfinite = orc.conv_silu(x, w, bias, prev)
    assert nonfinite == 0
    ref, mag = _conv_ref(x, w, bias, prev)
    # binary32 chain: each of the W fused steps rounds once (<= 2^-24 of the
    # running magnitude); silu's slope is below 1.1; then silu's own 4 ulp
    bound = 4 * _ulp(ref.astype(np.float32)) + 1.1 * W * 2.0 ** -24 * mag + 1e-30
    err = np.abs(u.astype(np.float64) - ref)
    assert np.all(err <= bound), "worst excess %.3g" % (err - bound).max()
    # the state of the next call: the last W - 1 inputs
    if W > 1:
        np.testing.assert_array_equal(st, x[..., L - (W - 1):])


@pytest.mark.parametrize("W,L1", [(4, 1), (4, 2), (4, 17), (3, 30), (2, 0)])
def test_conv_split_with_state(orc, W, L1):
    """A call on steps [0, L1) and one on [L1, L) with the first call's state
    give, bit for bit, the unsplit call (also when L1 < W - 1: the state then
    still holds inputs from before the first call)."""
    rng = np.random.default_rng(7 + W + L1)
    b, d, L = 2, 5, 40
    x = rng.standard_normal((b, d, L)).astype(np.float16)
    w = rng.standard_normal((d, W)).astype(np.float32)
    bias = rng.standard_normal(d).astype(np.float32)
    prev = rng.standard_normal((b, d, W - 1)).astype(np.float16)
    u, st, _ = orc.conv_silu(x, w, bias, prev)
    ua, sa, _ = orc.conv_silu(x[..., :L1], w, bias, prev)
    ub, sb, _ = orc.conv_silu(x[..., L1:], w, bias, sa)
    np.testing.assert_array_equal(np.concatenate([ua, ub], axis=-1), u)
    np.testing.assert_array_equal(sb, st)


def test_conv_nonfinite_counted(orc):
    x = np.zeros((1, 2, 8), np.float16)
    x[0, 1, 3] = np.inf
    u, _, nonfinite = orc.conv_silu(x, np.ones((2, 4), np.float32))
    assert nonfinite > 0 and np.all(np.isfinite(u[0, 0]))
