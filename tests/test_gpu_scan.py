"""GPU Mamba-1 W8A8 selective scan vs the oracle (Quamba2 abstract: W8A8
Mamba1 backbone; Quamba-SE write-up 2.2 for soft-edge x).

Tolerances: max |y - y_ref| <= 2e-3 max |y_ref| (y is stored as binary16),
final state relative L2 <= 1e-4."""
import numpy as np
import pytest
import torch

from gpu_util import Y_TOL, H, T, assert_scan_close, dev, status_word, y_err
from problems import m1_problem, oracle_kwargs
from quantized_state_space_b200 import _native as N
from quantized_state_space_b200 import api, calibrate, synth

pytestmark = pytest.mark.gpu


def gpu_scan(p, **kw):
    args = dict(D=T(p["D"]), z=T(p["z"]), dt_bias=T(p["dt_bias"]), h0=T(p.get("h0")))
    if p["x"].dtype == np.uint8:
        args["se_scale"] = p["se_scale"]
    else:
        args["x_group"] = T(p["x_group"])
        args["x_scale"] = T(p["x_scale"])
    args.update(kw)
    y, hf = api.selective_scan(T(p["x"]), T(p["dt"]), T(p["A"]), T(p["B"]), T(p["C"]),
                               T(p["B_scale"]), T(p["C_scale"]), p["state_group_size"], **args)
    return H(y).astype(np.float64), H(hf)


def oracle_scan(orc, p, **kw):
    return orc.m1_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["B_scale"], p["C_scale"],
                       p["state_group_size"], **oracle_kwargs(p), **kw)


CASES = [
    # (b, L, d, N, G, gs, gate, h0, bias, fmt)
    (2, 200, 40, 16, 1, 4, True, False, False, "int8"),      # ragged L, partial channel tile
    (1, 256, 64, 16, 1, 16, False, False, False, "int8"),    # the tiny workload's shape
    (3, 129, 48, 16, 2, 4, True, True, True, "int8"),        # G = 2, h0, bias, ragged
    (2, 64, 64, 4, 1, 2, True, True, False, "int8"),
    (2, 96, 40, 8, 2, 4, False, True, True, "int8"),
    (2, 80, 32, 32, 1, 8, True, True, False, "int8"),
    (1, 70, 24, 64, 1, 16, True, False, True, "int8"),
    (2, 192, 48, 16, 1, 4, True, True, False, "softedge"),
    (1, 17, 16, 16, 1, 4, True, False, False, "int8"),       # L < chunk, L % 16 != 0
    (1, 1, 16, 16, 1, 4, True, True, False, "int8"),         # one step
    (4, 512, 96, 16, 1, 4, True, False, False, "int8"),      # several chunks and tiles
]


@pytest.mark.parametrize("ci", range(len(CASES)))
def test_scan_vs_oracle(orc, ci):
    b, L, d, N_, G, gs, gate, h0, bias, fmt = CASES[ci]
    p = m1_problem(100 + ci, b, L, d, N_, G=G, gs=gs, gate=gate, h0=h0, bias=bias,
                   x_format=fmt)
    y, hf = gpu_scan(p)
    yo, ho = oracle_scan(orc, p)
    assert_scan_close(y, yo.reshape(y.shape), hf, ho.reshape(hf.shape))


def test_scan_softplus_off_and_delta_zero(orc):
    p = m1_problem(5, 2, 100, 32, 16, gate=False, h0=True)
    p["dt"][:] = 0
    y, hf = gpu_scan(p, dt_softplus=False)
    yo, ho = oracle_scan(orc, p, dt_softplus=False)
    assert_scan_close(y, yo.reshape(y.shape), hf, ho.reshape(hf.shape))
    np.testing.assert_array_equal(hf, p["h0"])  # delta = 0 keeps the state


def test_scan_empty_sequence():
    p = m1_problem(6, 2, 16, 16, 16, h0=True)
    x = T(np.zeros((2, 16, 0), np.int8))
    dt = T(np.zeros((2, 16, 0), np.float16))
    B = T(np.zeros((2, 1, 16, 0), np.int8))
    y, hf = api.selective_scan(x, dt, T(p["A"]), B, B, T(p["B_scale"]), T(p["C_scale"]), 4,
                               x_group=T(p["x_group"]), x_scale=T(p["x_scale"]), h0=T(p["h0"]))
    np.testing.assert_array_equal(H(hf), p["h0"])


def test_scan_bad_group_status():
    p = m1_problem(7, 1, 32, 16, 16)
    p["x_group"][3] = 99
    st = status_word()
    gpu_scan(p, status=st)
    assert int(H(st)[0]) & N.DEV_BAD_GROUP


def test_scan_channel_permutation_bit_exact():
    """Quamba2 compute invariance: permuting channels with their cluster ids,
    A, D, dt, z permutes y and the state exactly."""
    p = m1_problem(8, 2, 300, 64, 16, gate=True, h0=True, bias=True)
    perm = np.random.default_rng(1).permutation(64)
    q = dict(p)
    for k in ("x", "dt", "z"):
        q[k] = np.ascontiguousarray(p[k][:, perm, :])
    q["x_group"], q["A"], q["D"] = p["x_group"][perm], p["A"][perm], p["D"][perm]
    q["dt_bias"], q["h0"] = p["dt_bias"][perm], np.ascontiguousarray(p["h0"][:, perm, :])
    y, hf = gpu_scan(p)
    yq, hq = gpu_scan(q)
    np.testing.assert_array_equal(yq, y[:, perm, :])
    np.testing.assert_array_equal(hq, hf[:, perm, :])


def test_scan_power_of_two_scale_linearity():
    """Doubling every x scale doubles y and the state exactly (no gate,
    zero initial state): each product with x is an exact doubling."""
    p = m1_problem(9, 2, 256, 32, 16, gate=False)
    y, hf = gpu_scan(p)
    q = dict(p)
    q["x_scale"] = (p["x_scale"] * 2).astype(np.float32)
    y2, h2 = gpu_scan(q)
    # binary16 subnormals (|y| < 2^-14) round on an absolute grid, so the
    # doubling is exact only where y itself is a normal binary16 number
    normal = np.abs(y) >= 2.0 ** -14
    np.testing.assert_array_equal(y2[normal], 2 * y[normal])
    assert np.all(np.abs(y2[~normal] - 2 * y[~normal]) <= 2.0 ** -24)
    np.testing.assert_array_equal(h2, 2 * hf)


def test_scan_checkpoint_split_bit_exact():
    """scan(L) equals scan(first 256 steps) then scan(rest, h0 = that state)."""
    p = m1_problem(10, 2, 512, 32, 16, gate=True)
    y, hf = gpu_scan(p)
    a = dict(p)
    b = dict(p)
    for k in ("x", "dt", "z"):
        a[k] = np.ascontiguousarray(p[k][..., :256])
        b[k] = np.ascontiguousarray(p[k][..., 256:])
    for k in ("B", "C"):
        a[k] = np.ascontiguousarray(p[k][..., :256])
        b[k] = np.ascontiguousarray(p[k][..., 256:])
    ya, ha = gpu_scan(a)
    b["h0"] = ha
    yb, hb = gpu_scan(b)
    np.testing.assert_array_equal(np.concatenate([ya, yb], axis=-1), y)
    np.testing.assert_array_equal(hb, hf)


# ---- time segments: L cut into k segments scanned in parallel (later ones
# from a zero state) plus the carry-in pass; the recurrence is linear in the
# state, so the result is the one-pass result up to rounding

SEG_CASES = [
    # (b, L, d, N, G, gs, gate, h0, bias, fmt, k)
    (2, 200, 40, 16, 1, 4, True, False, False, "int8", 2),    # ragged L: short last segment
    (3, 512, 48, 16, 2, 4, True, True, True, "int8", 4),      # G = 2, h0, bias
    (2, 300, 32, 8, 1, 4, False, True, True, "int8", 3),
    (2, 256, 32, 32, 1, 8, True, True, False, "int8", 2),
    (1, 200, 24, 64, 1, 16, True, False, True, "int8", 3),
    (2, 384, 48, 16, 1, 4, True, True, False, "softedge", 3),
    (2, 96, 64, 4, 1, 2, True, True, False, "int8", 2),
    (1, 2048, 16, 16, 1, 4, True, True, True, "int8", 8),     # eight 256-step segments
]


@pytest.mark.parametrize("ci", range(len(SEG_CASES)))
def test_scan_time_segments_vs_oracle(orc, ci):
    b, L, d, N_, G, gs, gate, h0, bias, fmt, k = SEG_CASES[ci]
    p = m1_problem(400 + ci, b, L, d, N_, G=G, gs=gs, gate=gate, h0=h0, bias=bias,
                   x_format=fmt)
    y, hf = gpu_scan(p, time_segments=k)
    yo, ho = oracle_scan(orc, p)
    assert_scan_close(y, yo.reshape(y.shape), hf, ho.reshape(hf.shape))
    # and close to the one-pass kernel (y of later segments rounded twice)
    y1, h1 = gpu_scan(p)
    assert y_err(y, y1) <= 2 * 2.0 ** -11
    assert np.linalg.norm(hf - h1) <= 1e-5 * np.linalg.norm(h1)


def test_scan_time_segments_fused_encode_bit_exact():
    """Binary16 x encoded in the scan with time segments equals the separate
    quantizer followed by the code-reading scan with the same segments."""
    b, L, d, N_ = 2, 320, 48, 16
    p = m1_problem(450, b, L, d, N_, gate=True, h0=True)
    rng = np.random.default_rng(451)
    xf = _f16_activations(rng, (b, d, L))
    grp, xs = T(p["x_group"]), T(p["x_scale"])
    codes, _ = api.quantize_groups(T(xf), b, d, L, grp, int(xs.numel()), scales=xs)
    args = (T(p["dt"]), T(p["A"]), T(p["B"]), T(p["C"]), T(p["B_scale"]), T(p["C_scale"]), 4)
    kw = dict(x_group=grp, x_scale=xs, D=T(p["D"]), z=T(p["z"]), h0=T(p["h0"]), time_segments=3)
    y1, h1 = api.selective_scan(codes, *args, **kw)
    y2, h2 = api.selective_scan(T(xf), *args, **kw)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(H(y2).view(np.uint16), H(y1).view(np.uint16))
    np.testing.assert_array_equal(H(h2).view(np.uint32), H(h1).view(np.uint32))


def test_scan_time_segments_off_with_int8_y():
    """With the int8 y output the call keeps one pass: the bytes equal the
    call without segments."""
    p = m1_problem(460, 2, 256, 32, 16, gate=True, h0=True)
    yg = T(np.arange(32, dtype=np.int32) % 2)
    ys = T(np.array([0.02, 0.05], np.float32))
    args = (T(p["x"]), T(p["dt"]), T(p["A"]), T(p["B"]), T(p["C"]), T(p["B_scale"]),
            T(p["C_scale"]), 4)
    kw = dict(x_group=T(p["x_group"]), x_scale=T(p["x_scale"]), D=T(p["D"]), z=T(p["z"]),
              h0=T(p["h0"]), y_group=yg, y_scale=ys)
    a = api.selective_scan(*args, **kw)
    c = api.selective_scan(*args, time_segments=4, **kw)
    torch.cuda.synchronize()
    for u, v in zip(a, c):
        np.testing.assert_array_equal(H(u), H(v))


@pytest.mark.parametrize("cuts", [(0, 512), (0, 300, 301, 700)])
def test_m1_sequence_sharded_vs_oracle(orc, cuts):
    """Mamba-1 sequence sharding emulated in one process: each slice scanned
    from a zero state (the first from h0) with its per-(channel, state) log2
    decays, the summaries folded by the state-chain kernel, each later
    slice's carried start state added by the carry-in kernel; the
    concatenated y and the folded final state against the oracle's unsplit
    scan."""
    b, L, d, N_ = 2, 1000, 48, 16
    p = m1_problem(470, b, L, d, N_, gate=True, h0=True, bias=True)
    yo, ho = oracle_scan(orc, p)
    bounds = list(cuts) + [L]
    ys, h_ends, decs = [], [], []
    for r in range(len(bounds) - 1):
        sl = slice(bounds[r], bounds[r + 1])
        q = dict(p)
        for k in ("x", "dt", "z", "B", "C"):
            q[k] = np.ascontiguousarray(p[k][..., sl])
        args = (T(q["x"]), T(q["dt"]), T(q["A"]), T(q["B"]), T(q["C"]), T(q["B_scale"]),
                T(q["C_scale"]), p["state_group_size"])
        kw = dict(D=T(q["D"]), z=T(q["z"]), dt_bias=T(q["dt_bias"]))
        dec = torch.empty((b, d, N_), dtype=torch.float32, device=dev())
        y, he = api.selective_scan(*args, x_group=T(q["x_group"]), x_scale=T(q["x_scale"]),
                                   h0=T(p["h0"]) if r == 0 else None, dec_final=dec, **kw)
        # the log2 decays: A_cn log2(e) sum_t delta_t
        dv = q["dt"].astype(np.float64) + q["dt_bias"].astype(np.float64)[None, :, None]
        ref = (np.logaddexp(0.0, dv).sum(axis=2)[:, :, None] * q["A"].astype(np.float64)[None]
               * np.log2(np.e))
        np.testing.assert_allclose(H(dec), ref, rtol=2e-5, atol=1e-4)
        if r > 0:
            carry = api.state_chain(h_ends, decs)
            he_true = he.clone()  # the chain below folds the slices' local states
            api.selective_scan_carry_in(*args, carry, y, h_final=he_true, **kw)
        ys.append(H(y).astype(np.float64))
        h_ends.append(he)
        decs.append(dec)
    hf = H(api.state_chain(h_ends, decs))
    # the last carry-in's h_final: the same state as the fold of every slice
    np.testing.assert_allclose(H(he_true), hf, rtol=0, atol=1e-5 * np.abs(hf).max())
    y = np.concatenate(ys, axis=-1)
    assert_scan_close(y, yo.reshape(y.shape), hf, ho.reshape(hf.shape))


# ---- full-size workloads, end to end from raw activations ------------------

def _m1_end_to_end(orc, name, n_units=96, time_segments=1):
    dm, raw = synth.workload_inputs(name)
    b, L, d, Nst, G, gs = dm["batch"], dm["seqlen"], dm["dim"], dm["dstate"], dm["ngroups"], \
        dm["state_group_size"]
    gmap = calibrate.state_group_map(G, Nst, gs)
    # product: host calibration + GPU quantizers + GPU scan
    bs = calibrate.state_group_absmax_scales(raw["B"], G, Nst, gs, "gnl")
    cs = calibrate.state_group_absmax_scales(raw["C"], G, Nst, gs, "gnl")
    Bq, _ = api.quantize_groups(T(raw["B"]), b, G * Nst, L, T(gmap), G * Nst // gs, scales=T(bs))
    Cq, _ = api.quantize_groups(T(raw["C"]), b, G * Nst, L, T(gmap), G * Nst // gs, scales=T(cs))
    if name == "softedge":
        s, lo, hi = calibrate.softedge_params(raw["x"])
        xq = api.softedge_encode(T(raw["x"]), s, lo, hi, 2)
        xkw = dict(se_scale=s)
    else:
        k = dm["x_clusters"]
        if k == 1:
            xq, xs = api.quantize_groups(T(raw["x"]), b, d, L, T(np.zeros(d, np.int32)), 1,
                                         absmax=True)
            xkw = dict(x_group=T(np.zeros(d, np.int32)), x_scale=xs)
        else:
            grp, xs = calibrate.m1_x_clusters(raw["x"], k)
            xq, _ = api.quantize_groups(T(raw["x"]), b, d, L, T(grp), k, scales=T(xs))
            xkw = dict(x_group=T(grp), x_scale=T(xs))
    y, hf = api.selective_scan(xq, T(raw["dt"]), T(raw["A"]), Bq, Cq, T(bs), T(cs), gs,
                               D=T(raw["D"]), z=T(raw["z"]), time_segments=time_segments, **xkw)
    torch.cuda.synchronize()
    # oracle: its own calibration and quantizers from the same raw arrays; the
    # B/C scale index of row (g, n) is (g N + n) / gs in the ABI's layout
    gmap = np.arange(G * Nst) // gs
    _, obs, _ = orc.quantize_groups(raw["B"], b, G * Nst, L, gmap, G * Nst // gs, orc.SCALE_ABSMAX)
    _, ocs, _ = orc.quantize_groups(raw["C"], b, G * Nst, L, gmap, G * Nst // gs, orc.SCALE_ABSMAX)
    oB, _, _ = orc.quantize_groups(raw["B"], b, G * Nst, L, gmap, G * Nst // gs, orc.SCALE_STATIC, obs)
    oC, _, _ = orc.quantize_groups(raw["C"], b, G * Nst, L, gmap, G * Nst // gs, orc.SCALE_STATIC, ocs)
    np.testing.assert_array_equal(H(Bq), oB)
    np.testing.assert_array_equal(H(Cq), oC)
    if name == "softedge":
        olo = np.float32(orc.percentile_abs(raw["x"], 5.0))
        ohi = np.float32(orc.percentile_abs(raw["x"], 99.9))
        osc = np.float32(np.float64(ohi) / 63.0)
        ox, _ = orc.softedge_encode(raw["x"], osc, olo, ohi, 2)
        okw = dict(se_scale=float(osc))
    else:
        k = dm["x_clusters"]
        if k == 1:
            ox, oxs, _ = orc.quantize_groups(raw["x"], b, d, L, np.zeros(d, np.int32), 1,
                                             orc.SCALE_ABSMAX)
            okw = dict(x_group=np.zeros(d, np.int32), x_scale=oxs)
        else:
            og, oxs = orc.cluster_by_absmax(orc.absmax_per_mid(raw["x"], b, d, L), k)
            ox, _, _ = orc.quantize_groups(raw["x"], b, d, L, og, k, orc.SCALE_STATIC, oxs)
            okw = dict(x_group=og, x_scale=oxs)
    np.testing.assert_array_equal(H(xq), ox)
    rng = np.random.default_rng(0)
    units = rng.choice(b * d, size=min(n_units, b * d), replace=False)
    if raw.get("outlier_channels") is not None:  # always include the outlier channels
        units = np.unique(np.concatenate([units, raw["outlier_channels"]]))
    yo, ho = orc.m1_scan(ox, raw["dt"], raw["A"], oB, oC, obs, ocs, gs, D=raw["D"], z=raw["z"],
                         units=units, **okw)
    yg = H(y).reshape(b * d, L)[units].astype(np.float64)
    hg = H(hf).reshape(b * d, Nst)[units]
    # the tolerance is relative to max |y_ref| over the sampled channels
    e = assert_scan_close(yg, yo, hg, ho)
    # A few huge values set that max: the m130m outlier channels (x50 at
    # every step) and the softedge spikes (x100..1000 at single elements).
    # The same bound must also hold for the ordinary channels / positions
    # against their own max |y_ref|, or an error of several percent of a
    # typical |y| could pass.
    keep = np.ones(yo.shape, dtype=bool)
    if raw.get("outlier_channels") is not None:
        keep &= ~np.isin(units % d, raw["outlier_channels"])[:, None]
    if raw.get("spike_positions") is not None:
        flat = units[:, None] * L + np.arange(L)[None, :]  # (b, d, L) element index
        keep &= ~np.isin(flat, raw["spike_positions"])
    if not keep.all():
        assert keep.any()
        e2 = y_err(yg[keep], yo[keep])
        assert e2 <= Y_TOL, "ordinary channels / positions: y error %.3g > %.1g" % (e2, Y_TOL)
    return e


def test_tiny_workload_end_to_end(orc):
    _m1_end_to_end(orc, "tiny", n_units=64)


def test_m130m_workload_end_to_end(orc):
    _m1_end_to_end(orc, "m130m")


def test_softedge_workload_end_to_end(orc):
    _m1_end_to_end(orc, "softedge", n_units=64)


@pytest.mark.parametrize("k", [2, 4])
def test_m130m_workload_time_segments(orc, k):
    _m1_end_to_end(orc, "m130m", time_segments=k)


# ---- encode then scan: binary16 x encoded inside the scan (producer-side
# fusion; Quamba-SE write-up 4.1: the range check inside quantisation).  The fused call must equal the separate encoder followed by
# the code-reading scan, byte for byte, status word included.

FUSED_CASES = [
    # (b, L, d, N, G, gs, gate, h0, fmt)
    (2, 200, 40, 16, 1, 4, True, False, "group"),     # ragged L (no 16-byte rows), partial tile
    (2, 256, 64, 16, 2, 4, True, True, "group"),
    (2, 96, 64, 4, 1, 2, False, True, "group"),
    (1, 64, 16, 64, 1, 16, True, False, "group"),
    (2, 160, 48, 16, 1, 4, True, True, "softedge"),
    (1, 70, 32, 8, 1, 4, False, False, "softedge"),
]


def _f16_activations(rng, shape, outliers=True):
    x = rng.standard_normal(shape).astype(np.float32)
    if outliers:
        idx = rng.choice(x.size, size=max(1, x.size // 2000), replace=False)
        x.reshape(-1)[idx] *= rng.uniform(20, 200, size=idx.size)
    return x.astype(np.float16)


@pytest.mark.parametrize("ci", range(len(FUSED_CASES)))
def test_fused_encode_scan_bit_exact(ci):
    b, L, d, N_, G, gs, gate, h0, fmt = FUSED_CASES[ci]
    p = m1_problem(700 + ci, b, L, d, N_, G=G, gs=gs, gate=gate, h0=h0)
    rng = np.random.default_rng(750 + ci)
    xf = _f16_activations(rng, (b, d, L))
    xf.reshape(-1)[rng.choice(xf.size, size=3, replace=False)] = [np.inf, -np.inf, np.nan]
    xt = T(xf)
    common = dict(D=T(p["D"]), z=T(p["z"]), h0=T(p.get("h0")))
    args = (T(p["dt"]), T(p["A"]), T(p["B"]), T(p["C"]), T(p["B_scale"]), T(p["C_scale"]), gs)
    s_sep, s_fused = status_word(), status_word()
    if fmt == "group":
        grp = T(p["x_group"])
        xs = T(p["x_scale"])
        codes, _ = api.quantize_groups(xt, b, d, L, grp, int(xs.numel()), scales=xs, status=s_sep)
        y1, h1 = api.selective_scan(codes, *args, x_group=grp, x_scale=xs, status=s_sep, **common)
        y2, h2 = api.selective_scan(xt, *args, x_group=grp, x_scale=xs, status=s_fused, **common)
    else:
        finite = np.abs(xf[np.isfinite(xf)].astype(np.float64))
        lo, hi = float(np.percentile(finite, 5)), float(np.percentile(finite, 99.9))
        s = float(np.float32(hi / 63))
        codes = api.softedge_encode(xt, s, lo, hi, 2, status=s_sep)
        y1, h1 = api.selective_scan(codes, *args, se_scale=s, status=s_sep, **common)
        y2, h2 = api.selective_scan(xt, *args, se_scale=s, se_lo=lo, se_hi=hi, status=s_fused,
                                    **common)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(H(y2).view(np.uint16), H(y1).view(np.uint16))
    np.testing.assert_array_equal(H(h2).view(np.uint32), H(h1).view(np.uint32))
    assert int(H(s_fused)[0]) == int(H(s_sep)[0]) and int(H(s_fused)[0]) & 1  # NONFINITE seen


def test_fused_encode_scan_vs_oracle(orc):
    """The fused path against the oracle's quantizer followed by its scan."""
    b, L, d, N_, gs = 2, 300, 48, 16, 4
    p = m1_problem(790, b, L, d, N_, gs=gs, gate=True, h0=True, bias=True)
    rng = np.random.default_rng(791)
    xf = _f16_activations(rng, (b, d, L))
    y, hf = api.selective_scan(T(xf), T(p["dt"]), T(p["A"]), T(p["B"]), T(p["C"]),
                               T(p["B_scale"]), T(p["C_scale"]), gs, x_group=T(p["x_group"]),
                               x_scale=T(p["x_scale"]), D=T(p["D"]), z=T(p["z"]),
                               dt_bias=T(p["dt_bias"]), h0=T(p["h0"]))
    k = int(p["x_scale"].size)
    q, _, _ = orc.quantize_groups(xf, b, d, L, p["x_group"], k, orc.SCALE_STATIC, p["x_scale"])
    po = dict(p, x=q.reshape(b, d, L))
    yo, ho = oracle_scan(orc, po)
    assert_scan_close(H(y).astype(np.float64), yo.reshape(y.shape), H(hf), ho.reshape(hf.shape))


# ---- persistent-INT8 epilogue (SSDi8 abstract): int8 y with static per-cluster
# output scales; the bytes must equal the quantizer applied to the binary16 y.

YQ_CASES = [
    # (b, L, d, N, gs, fmt)
    (2, 256, 64, 16, 4, "int8"),
    (2, 200, 40, 16, 4, "int8"),      # ragged L: scalar stores
    (1, 96, 64, 4, 2, "int8"),
    (1, 64, 16, 64, 16, "softedge"),
]


@pytest.mark.parametrize("ci", range(len(YQ_CASES)))
def test_scan_int8_y_bit_exact(orc, ci):
    b, L, d, N_, gs, fmt = YQ_CASES[ci]
    p = m1_problem(800 + ci, b, L, d, N_, gs=gs, gate=True, h0=True, x_format=fmt)
    rng = np.random.default_rng(820 + ci)
    ky = 4
    ygrp = rng.integers(0, ky, size=d).astype(np.int32)
    ygrp[3] = ky + 5                                   # one channel with a bad cluster id
    ysc = synth.random_scales(rng, ky, 0.002, 0.02)
    st = status_word()
    y, hf, yq = (None, None, None)
    y_t, hf_t, yq_t = api.selective_scan(
        T(p["x"]), T(p["dt"]), T(p["A"]), T(p["B"]), T(p["C"]), T(p["B_scale"]), T(p["C_scale"]),
        gs, y_group=T(ygrp), y_scale=T(ysc), status=st,
        **({"se_scale": p["se_scale"]} if fmt == "softedge" else
           {"x_group": T(p["x_group"]), "x_scale": T(p["x_scale"])}),
        D=T(p["D"]), z=T(p["z"]), h0=T(p["h0"]))
    ref, _ = api.quantize_groups(y_t, b, d, L, T(ygrp), ky, scales=T(ysc))
    np.testing.assert_array_equal(H(yq_t), H(ref))
    assert int(H(st)[0]) & 2                           # SSMQ_DEV_BAD_GROUP seen
    assert not H(yq_t)[:, 3].any()
    # without the binary16 y: same codes, same state
    y2, hf2, yq2 = api.selective_scan(
        T(p["x"]), T(p["dt"]), T(p["A"]), T(p["B"]), T(p["C"]), T(p["B_scale"]), T(p["C_scale"]),
        gs, y_group=T(ygrp), y_scale=T(ysc), want_y=False,
        **({"se_scale": p["se_scale"]} if fmt == "softedge" else
           {"x_group": T(p["x_group"]), "x_scale": T(p["x_scale"])}),
        D=T(p["D"]), z=T(p["z"]), h0=T(p["h0"]))
    assert y2 is None
    np.testing.assert_array_equal(H(yq2), H(yq_t))
    np.testing.assert_array_equal(H(hf2).view(np.uint32), H(hf_t).view(np.uint32))
    # the dequantized codes against the oracle's y: within the y tolerance plus half a step
    yo, _ = oracle_scan(orc, p)
    yo = yo.reshape(b, d, L)
    deq = H(yq_t).astype(np.float64) * ysc[np.clip(ygrp, 0, ky - 1)][None, :, None]
    ok = ygrp < ky
    lim = 2e-3 * np.abs(yo).max() + 0.5 * ysc[np.clip(ygrp, 0, ky - 1)][None, :, None]
    inside = np.abs(yo) <= 127 * ysc[np.clip(ygrp, 0, ky - 1)][None, :, None]
    assert np.all((np.abs(deq - yo) <= lim)[:, ok][inside[:, ok]])
