"""The fused producer of the scan input (causal depthwise conv + SiLU +
group quantizer / soft-edge encoder) against the oracle: the binary32 values
u, the codes and the carried conv state bit for bit, on ragged and
vectorised shapes, every width, both code formats, the range ends of the
exponential, non-finite inputs, split calls with the state, and the full-size
Mamba-130M and soft-edge layer shapes."""
import numpy as np
import pytest
import torch

from gpu_util import H, T, status_word
from quantized_state_space_b200 import _native as N
from quantized_state_space_b200 import api

pytestmark = pytest.mark.gpu


def _inputs(seed, b, d, L, W, bias=True, prev=True, outliers=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((b, d, L)).astype(np.float32)
    if outliers and d >= 8:
        x[:, rng.choice(d, size=max(1, d // 64), replace=False), :] *= 50.0
    w = rng.uniform(-0.6, 0.6, size=(d, W)).astype(np.float32)
    bs = rng.uniform(-0.5, 0.5, size=d).astype(np.float32) if bias else None
    xp = rng.standard_normal((b, d, W - 1)).astype(np.float16) if prev and W > 1 else None
    return x.astype(np.float16), w, bs, xp


def _oracle_codes(orc, u, fmt, k, rng_seed):
    """Calibration from the oracle's own u (offline step), then the oracle's
    quantizer / encoder on the binary32 u."""
    b, d, L = u.shape
    if fmt == "group":
        grp, sc = orc.cluster_by_absmax(orc.absmax_per_mid(u, b, d, L), k)
        codes, _, _ = orc.quantize_groups(u, b, d, L, grp, k, orc.SCALE_STATIC, sc)
        return codes, dict(x_group=grp, x_scale=sc)
    a = np.abs(u[np.isfinite(u)]).astype(np.float64)
    lo, hi = np.float32(np.percentile(a, 5)), np.float32(np.percentile(a, 99.9))
    s = np.float32(np.float64(hi) / 63.0)
    codes, _ = orc.softedge_encode(u, s, lo, hi, 2)
    return codes, dict(se_scale=float(s), se_lo=float(lo), se_hi=float(hi))


def _gpu(x, w, bs, xp, kw, want_u=True):
    kwt = {k: (T(v) if isinstance(v, np.ndarray) else v) for k, v in kw.items()}
    st = status_word()
    codes, u, state = api.conv_silu_quantize(T(x), T(w), bias=T(bs), x_prev=T(xp), want_u=True,
                                             want_state=True, status=st, **kwt)
    torch.cuda.synchronize()
    return H(codes), H(u), H(state), int(H(st)[0])


CASES = [
    # (b, d, L, W, bias, prev, fmt, k)
    (2, 24, 64, 4, True, True, "group", 4),      # vectorised rows, several vectors per row
    (2, 24, 70, 4, True, True, "group", 4),      # ragged rows: element path
    (1, 40, 16, 4, False, True, "group", 8),     # one vector per row (state in and out)
    (3, 17, 48, 3, True, False, "group", 3),
    (2, 32, 96, 2, True, True, "softedge", 1),
    (1, 16, 33, 1, True, False, "softedge", 1),  # width 1: no state
    (2, 64, 1024, 4, True, True, "group", 8),    # many vectors, grid-stride loop
    (1, 8, 5, 4, True, True, "softedge", 1),     # L < 16
]


@pytest.mark.parametrize("ci", range(len(CASES)))
def test_conv_silu_quantize_vs_oracle(orc, ci):
    b, d, L, W, bias, prev, fmt, k = CASES[ci]
    x, w, bs, xp = _inputs(300 + ci, b, d, L, W, bias, prev)
    uo, so, nf = orc.conv_silu(x, w, bs, xp)
    assert nf == 0
    co, kw = _oracle_codes(orc, uo, fmt, k, ci)
    codes, u, state, status = _gpu(x, w, bs, xp, kw)
    np.testing.assert_array_equal(u.view(np.uint32), uo.view(np.uint32))
    np.testing.assert_array_equal(codes.view(np.uint8), co.view(np.uint8))
    if W > 1:
        np.testing.assert_array_equal(state.view(np.uint16), so.view(np.uint16))
    assert status == 0


def test_range_ends_and_nonfinite(orc):
    """|a| above 87 (the exponential's range ends, scalar route), exact zeros,
    and non-finite inputs (coded 0, NONFINITE raised) in vectorised rows."""
    b, d, L, W = 1, 8, 64, 4
    x, w, bs, xp = _inputs(55, b, d, L, W, outliers=False)
    x = x.astype(np.float32)
    x[0, 0, 10:20] = 400.0    # a > 87: e underflows to 0, u = a
    x[0, 1, 5:12] = -400.0    # a < -87: e = inf, u = -0
    x[0, 2, 30:34] = 60.0     # a near the boundary
    x[0, 3, :] = 0.0          # a = bias
    x[0, 4, 40] = np.inf
    x[0, 5, 3] = np.nan
    x = x.astype(np.float16)
    w[:] = np.abs(w) + 0.1
    uo, so, nf = orc.conv_silu(x, w, bs, xp)
    assert nf > 0
    grp = np.arange(d, dtype=np.int32) % 2
    sc = np.array([0.05, 2.0], np.float32)
    co, _, _ = orc.quantize_groups(uo, b, d, L, grp, 2, orc.SCALE_STATIC, sc)
    codes, u, state, status = _gpu(x, w, bs, xp, dict(x_group=grp, x_scale=sc))
    # NaN payloads differ between implementations: NaN where the oracle has
    # NaN, every other value bit for bit (infinities and signed zeros too)
    nan = np.isnan(uo)
    assert nan.any() and np.array_equal(np.isnan(u), nan)
    np.testing.assert_array_equal(u[~nan].view(np.uint32), uo[~nan].view(np.uint32))
    np.testing.assert_array_equal(codes, co)
    assert status & N.DEV_NONFINITE


@pytest.mark.parametrize("L1", [0, 16, 48, 5])
def test_split_with_state_bit_exact(orc, L1):
    """Steps [0, L1) and then [L1, L) with the first call's state give the
    unsplit call's codes, values and state."""
    b, d, L, W = 2, 16, 128, 4
    x, w, bs, xp = _inputs(77 + L1, b, d, L, W)
    grp = (np.arange(d) % 4).astype(np.int32)
    sc = np.array([0.01, 0.02, 0.05, 0.1], np.float32)
    kw = dict(x_group=T(grp), x_scale=T(sc))
    c, u, s = api.conv_silu_quantize(T(x), T(w), bias=T(bs), x_prev=T(xp), want_u=True,
                                     want_state=True, **kw)
    ca, ua, sa = api.conv_silu_quantize(T(x[..., :L1]), T(w), bias=T(bs), x_prev=T(xp),
                                        want_u=True, want_state=True, **kw)
    cb, ub, sb = api.conv_silu_quantize(T(x[..., L1:]), T(w), bias=T(bs), x_prev=sa,
                                        want_u=True, want_state=True, **kw)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(np.concatenate([H(ca), H(cb)], -1), H(c))
    np.testing.assert_array_equal(np.concatenate([H(ua), H(ub)], -1).view(np.uint32),
                                  H(u).view(np.uint32))
    np.testing.assert_array_equal(H(sb).view(np.uint16), H(s).view(np.uint16))


def test_empty_and_state_only():
    """L = 0: no codes; the state passes through."""
    b, d, W = 2, 8, 4
    rng = np.random.default_rng(9)
    xp = rng.standard_normal((b, d, W - 1)).astype(np.float16)
    w = rng.standard_normal((d, W)).astype(np.float32)
    grp = np.zeros(d, np.int32)
    c, s = api.conv_silu_quantize(T(np.zeros((b, d, 0), np.float16)), T(w), x_prev=T(xp),
                                  x_group=T(grp), x_scale=T(np.ones(1, np.float32)),
                                  want_state=True)
    torch.cuda.synchronize()
    assert c.numel() == 0
    np.testing.assert_array_equal(H(s).view(np.uint16), xp.view(np.uint16))


@pytest.mark.parametrize("name", ["m130m", "softedge"])
def test_full_size_layer(orc, name):
    """Full-size channel-major layers: the Mamba-130M-shaped layer (8 x 1536 x
    2048, 8 clusters, int8 codes) and the soft-edge layer (16 x 1536 x 8192,
    soft-edge codes; batch rows 0 and 15 checked).  The conv input is seeded
    like the workloads' x (outlier channels x50 for m130m, Student-t(3) with
    sparse spikes for softedge)."""
    from quantized_state_space_b200 import synth
    dm, raw = synth.workload_inputs(name)
    x = raw["x"]
    b, d, L = x.shape
    W = 4
    rng = np.random.default_rng(12)
    w = rng.uniform(-0.5, 0.5, size=(d, W)).astype(np.float32)
    bs = rng.uniform(-0.2, 0.2, size=d).astype(np.float32)
    rows = slice(None) if name == "m130m" else [0, b - 1]
    xs = np.ascontiguousarray(x[rows])
    uo, so, _ = orc.conv_silu(xs, w, bs)
    if name == "m130m":
        grp, sc = orc.cluster_by_absmax(orc.absmax_per_mid(uo, b, d, L), 8)
        co, _, _ = orc.quantize_groups(uo, b, d, L, grp, 8, orc.SCALE_STATIC, sc)
        kw = dict(x_group=T(grp), x_scale=T(sc))
    else:
        a = np.abs(uo[np.isfinite(uo)]).astype(np.float64)
        lo, hi = np.float32(np.percentile(a, 5)), np.float32(np.percentile(a, 99.9))
        s = np.float32(np.float64(hi) / 63.0)
        co, _ = orc.softedge_encode(uo, s, lo, hi, 2)
        kw = dict(se_scale=float(s), se_lo=float(lo), se_hi=float(hi))
    st = status_word()
    codes, state = api.conv_silu_quantize(T(x), T(w), bias=T(bs), want_state=True, status=st,
                                          **kw)
    torch.cuda.synchronize()
    got = H(codes)[rows]
    np.testing.assert_array_equal(got.view(np.uint8), co.view(np.uint8))
    np.testing.assert_array_equal(H(state)[rows].view(np.uint16), so.view(np.uint16))
    assert int(H(st)[0]) == 0
