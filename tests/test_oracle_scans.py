"""Pins of the oracle's scans against closed forms, brute-force materialised
sums, the quadratic (attention) dual form built from numpy matmuls, and
identities between the three forms.

Recurrence (the Mamba selective SSM that Quamba2 and SSDi8 quantize):
    h_t = exp(delta_t A) h_{t-1} + delta_t B_t x_t,  y_t = C_t . h_t + D x_t
    (optionally y_t *= silu(z_t)), delta_t = softplus(dt_t + bias).
"""
import numpy as np
import pytest
from scipy.special import expit

from problems import m1_problem, oracle_kwargs, ssd_problem

# ---- numpy restatements used as independent references ----------------------


def _deq_x_m1(p):
    return p["x"].astype(np.float64) * p["x_scale"][p["x_group"]].astype(np.float64)[None, :, None]


def _deq_bc(q, scale, gs, axis_n):
    """int8 B/C times its state-group scale; scale index g * (N/gs) + n // gs."""
    q = q.astype(np.float64)
    G_axis = axis_n - 1
    G, N = q.shape[G_axis], q.shape[axis_n]
    s = scale.astype(np.float64).reshape(G, N // gs)
    s = np.repeat(s, gs, axis=1)  # (G, N)
    shape = [1] * q.ndim
    shape[G_axis], shape[axis_n] = G, N
    return q * s.reshape(shape)


def _delta(dt, bias, softplus):
    v = dt.astype(np.float64)
    if bias is not None:
        v = v + bias
    return np.logaddexp(0.0, v) if softplus else v


def m1_bruteforce(p, softplus=True):
    """Unrolled solution of the Mamba-1 recurrence:
    y_t = sum_n C_tn [sum_{s<=t} exp(A_n (cum_t - cum_s)) d_s B_sn x_s
                      + exp(A_n cum_t) h0_n] + D x_t."""
    x = _deq_x_m1(p)
    b, d, L = x.shape
    Bq, Cq = p["B"], p["C"]
    G, N = Bq.shape[1], Bq.shape[2]
    Bv = _deq_bc(Bq, p["B_scale"], p["state_group_size"], 2)
    Cv = _deq_bc(Cq, p["C_scale"], p["state_group_size"], 2)
    bias = None if p["dt_bias"] is None else p["dt_bias"].astype(np.float64)[None, :, None]
    dl = _delta(p["dt"], bias, softplus)
    y = np.zeros((b, d, L))
    hf = np.zeros((b, d, N))
    tri = np.tril(np.ones((L, L), bool))
    for bb in range(b):
        for c in range(d):
            g = c * G // d
            cum = np.cumsum(dl[bb, c])
            A = p["A"][c].astype(np.float64)
            expo = A[None, None, :] * (cum[:, None, None] - cum[None, :, None])  # t,s,n
            dec = np.where(tri[:, :, None], np.exp(np.minimum(expo, 0.0)), 0.0)
            src = dl[bb, c][:, None] * Bv[bb, g].T * x[bb, c][:, None]  # s,n
            h = np.einsum("tsn,sn->tn", dec, src)
            if p.get("h0") is not None:
                h = h + np.exp(A[None, :] * cum[:, None]) * p["h0"][bb, c].astype(np.float64)
            yy = np.sum(Cv[bb, g].T * h, axis=1) + p["D"][c] * x[bb, c]
            if p["z"] is not None:
                zz = p["z"][bb, c].astype(np.float64)
                yy = yy * zz * expit(zz)
            y[bb, c] = yy
            hf[bb, c] = h[-1]
    return y, hf


def ssd_dual(p, softplus=True):
    """Quadratic (attention) form of SSD per (b, h): with S = cumsum(delta A),
    Y = (tril(C B^T * exp(S_t - S_s)) * delta_s) X + exp(S) (C h0^T) + D X."""
    b, L, H, P = p["x"].shape
    G, N = p["B"].shape[2], p["B"].shape[3]
    x = p["x"].astype(np.float64) * p["x_scale"][p["x_group"]].astype(np.float64).reshape(1, 1, H, P)
    Bv = _deq_bc(p["B"], p["B_scale"], p["state_group_size"], 3)
    Cv = _deq_bc(p["C"], p["C_scale"], p["state_group_size"], 3)
    bias = None if p["dt_bias"] is None else p["dt_bias"].astype(np.float64)[None, None, :]
    dl = _delta(p["dt"], bias, softplus)
    y = np.zeros((b, H, L, P))
    hf = np.zeros((b, H, P, N))
    for bb in range(b):
        for h in range(H):
            g = h * G // H
            S = np.cumsum(dl[bb, :, h] * float(p["A"][h]))
            CB = Cv[bb, :, g, :] @ Bv[bb, :, g, :].T
            M = np.tril(CB * np.exp(np.minimum(S[:, None] - S[None, :], 0.0))) * dl[bb, :, h][None, :]
            X = x[bb, :, h, :]
            Y = M @ X + float(p["D"][h]) * X
            W = np.exp(S[-1] - S) * dl[bb, :, h]  # weight of each step in the final state
            H_f = (X * W[:, None]).T @ Bv[bb, :, g, :]
            if p.get("h0") is not None:
                h0 = p["h0"][bb, h].astype(np.float64)
                Y = Y + np.exp(S)[:, None] * (Cv[bb, :, g, :] @ h0.T)
                H_f = H_f + np.exp(S[-1]) * h0
            if p["z"] is not None:
                zz = p["z"][bb, :, h, :].astype(np.float64)
                Y = Y * zz * expit(zz)
            y[bb, h] = Y
            hf[bb, h] = H_f
    return y, hf


def _m1(orc, p, **kw):
    return orc.m1_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["B_scale"], p["C_scale"],
                       p["state_group_size"], **oracle_kwargs(p), **kw)


def _ssd(orc, p, **kw):
    return orc.ssd_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["B_scale"], p["C_scale"],
                        p["state_group_size"], **oracle_kwargs(p), **kw)


def _rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# ---- Mamba-1 ----------------------------------------------------------------

@pytest.mark.parametrize("gate,h0,bias,G,gs", [(True, False, False, 1, 4), (False, True, True, 2, 8),
                                              (True, True, False, 4, 2)])
def test_m1_bruteforce(orc, gate, h0, bias, G, gs):
    p = m1_problem(1, 2, 40, 8, 16, G=G, gs=gs, gate=gate, h0=h0, bias=bias, dt_mean=-1.0)
    y, hf = _m1(orc, p)
    yb, hb = m1_bruteforce(p)
    assert _rel(y.reshape(yb.shape), yb) < 1e-12
    assert _rel(hf.reshape(hb.shape), hb) < 1e-12


def test_m1_delta_zero_closed_form(orc):
    """delta = 0: the state never moves, y_t = C_t . h0 + D x_t."""
    p = m1_problem(2, 2, 33, 6, 16, gate=False, h0=True)
    p["dt"][:] = 0
    y, hf = _m1(orc, p, dt_softplus=False)
    x = _deq_x_m1(p)
    Cv = _deq_bc(p["C"], p["C_scale"], 4, 2)
    want = np.einsum("bnt,bdn->bdt", Cv[:, 0], p["h0"].astype(np.float64)) + p["D"][None, :, None] * x
    assert _rel(y.reshape(want.shape), want) < 1e-13
    np.testing.assert_array_equal(hf.reshape(p["h0"].shape), p["h0"].astype(np.float64))


def test_m1_lti_geometric_series(orc):
    """Constant inputs: h_t = a^(t+1) h0 + beta (1 - a^(t+1)) / (1 - a),
    a = exp(delta A_n), beta = delta B_n x."""
    p = m1_problem(3, 1, 50, 4, 16, gate=False, h0=True)
    L = 50
    p["dt"][:] = np.float16(0.0625)
    p["x"][:] = p["x"][:, :, :1]
    p["B"][:] = p["B"][:, :, :, :1]
    p["C"][:] = p["C"][:, :, :, :1]
    y, hf = _m1(orc, p, dt_softplus=False)
    x = _deq_x_m1(p)[0, :, 0]
    Bv = _deq_bc(p["B"], p["B_scale"], 4, 2)[0, 0, :, 0]
    Cv = _deq_bc(p["C"], p["C_scale"], 4, 2)[0, 0, :, 0]
    t = np.arange(1, L + 1)[:, None]
    for c in range(4):
        a = np.exp(0.0625 * p["A"][c].astype(np.float64))
        beta = 0.0625 * Bv * x[c]
        h = a[None, :] ** t * p["h0"][0, c] + beta[None, :] * (1 - a[None, :] ** t) / (1 - a[None, :])
        want = h @ Cv + p["D"][c] * x[c]
        assert _rel(y[c], want) < 1e-12
        assert _rel(hf[c], h[-1]) < 1e-12


def test_m1_lti_materialised_convolution(orc):
    """LTI system (constant delta, B, C) driven by a varying x: y is the causal
    convolution of x with the materialised kernel
    K_k = sum_n C_n exp(delta A_n)^k delta B_n, plus D x (numpy.convolve)."""
    L, d, delta = 64, 3, 0.0625
    p = m1_problem(4, 1, L, d, 16, gate=False, h0=False)
    p["dt"][:] = np.float16(delta)
    p["B"][:] = p["B"][:, :, :, :1]
    p["C"][:] = p["C"][:, :, :, :1]
    y, _ = _m1(orc, p, dt_softplus=False)
    gs = p["state_group_size"]
    x = _deq_x_m1(p)[0]
    Bv = _deq_bc(p["B"], p["B_scale"], gs, 2)[0, 0, :, 0]
    Cv = _deq_bc(p["C"], p["C_scale"], gs, 2)[0, 0, :, 0]
    k = np.arange(L)[:, None]
    for c in range(d):
        a = np.exp(delta * p["A"][c].astype(np.float64))
        K = (a[None, :] ** k * (delta * Bv)[None, :]) @ Cv
        want = np.convolve(x[c], K)[:L] + p["D"][c] * x[c]
        assert _rel(y[c], want) < 1e-12


def test_m1_softedge_bruteforce(orc):
    """x given as soft-edge codes: the scan equals the recurrence run on the
    decoded values (decoded here through the binary32 decoder, hence the
    1e-6 relative slack for its one rounding)."""
    p = m1_problem(4, 1, 30, 6, 16, gate=True, x_format="softedge", dt_mean=-2.0)
    y, _ = _m1(orc, p)
    xv = orc.softedge_decode(p["x"], p["se_scale"], 2).astype(np.float64)
    dl = _delta(p["dt"], None, True)
    Bv = _deq_bc(p["B"], p["B_scale"], 4, 2)
    Cv = _deq_bc(p["C"], p["C_scale"], 4, 2)
    ref = np.zeros((6, 30))
    for c in range(6):
        h = np.zeros(16)
        for t in range(30):
            h = np.exp(dl[0, c, t] * p["A"][c].astype(np.float64)) * h + dl[0, c, t] * Bv[0, 0, :, t] * xv[0, c, t]
            yy = Cv[0, 0, :, t] @ h + p["D"][c] * xv[0, c, t]
            zz = float(p["z"][0, c, t])
            ref[c, t] = yy * zz * expit(zz)
    assert _rel(y, ref) < 1e-6


def test_m1_channel_permutation_invariance(orc):
    """Quamba2's compute invariance: permuting channels together with their
    cluster map, A, D and dt permutes y and the state, bit for bit."""
    p = m1_problem(5, 2, 24, 12, 16, gate=True, h0=True, bias=True)
    perm = np.random.default_rng(0).permutation(12)
    q = dict(p)
    for k in ("x", "dt", "z"):
        q[k] = p[k][:, perm, :]
    q["x_group"] = p["x_group"][perm]
    q["A"], q["D"], q["dt_bias"] = p["A"][perm], p["D"][perm], p["dt_bias"][perm]
    q["h0"] = p["h0"][:, perm, :]
    y, hf = _m1(orc, p)
    yq, hq = _m1(orc, q)
    np.testing.assert_array_equal(yq.reshape(2, 12, -1), y.reshape(2, 12, -1)[:, perm, :])
    np.testing.assert_array_equal(hq.reshape(2, 12, -1), hf.reshape(2, 12, -1)[:, perm, :])


def test_m1_units_and_threads(orc):
    p = m1_problem(6, 3, 20, 8, 16)
    y, hf = _m1(orc, p, threads=1)
    y8, hf8 = _m1(orc, p, threads=8)
    np.testing.assert_array_equal(y, y8)
    units = np.array([23, 0, 9, 17])
    yu, hu = _m1(orc, p, units=units)
    np.testing.assert_array_equal(yu, y[units])
    np.testing.assert_array_equal(hu, hf[units])


def test_m1_split_with_h0(orc):
    """scan(L) equals scan(first half) followed by scan(second half) from its state."""
    p = m1_problem(7, 2, 40, 6, 16, gate=True)
    y, hf = _m1(orc, p)
    a = {k: (v[..., :20] if isinstance(v, np.ndarray) and v.ndim >= 3 and v.shape[-1] == 40 else v)
         for k, v in p.items()}
    b = {k: (v[..., 20:] if isinstance(v, np.ndarray) and v.ndim >= 3 and v.shape[-1] == 40 else v)
         for k, v in p.items()}
    ya, ha = _m1(orc, a)
    b["h0"] = ha.reshape(2, 6, 16).astype(np.float32)
    yb, hb = _m1(orc, b)
    assert _rel(ya, y[:, :20]) < 1e-15
    # the split rounds the carried state to float32 once
    assert _rel(yb, y[:, 20:]) < 1e-6
    assert _rel(hb, hf) < 1e-6


# ---- SSD ----------------------------------------------------------------------

@pytest.mark.parametrize("G,gate,h0,bias", [(1, False, False, False), (2, True, True, True)])
def test_ssd_dual_form(orc, G, gate, h0, bias):
    p = ssd_problem(11, 2, 48, 4, 8, 16, G=G, gs=4, gate=gate, h0=h0, bias=bias, dt_mean=-1.5)
    y, hf = _ssd(orc, p)
    yd, hd = ssd_dual(p)
    assert _rel(y.reshape(2, 4, 48, 8), yd) < 1e-12
    assert _rel(hf.reshape(hd.shape), hd) < 1e-12


@pytest.mark.parametrize("chunk", [1, 7, 16, 64, 100])
def test_ssd_chunked_equals_sequential(orc, chunk):
    p = ssd_problem(12, 2, 64, 3, 8, 16, G=1, gs=8, gate=True, h0=True, bias=True, dt_mean=-2.0)
    y, hf = _ssd(orc, p)
    yc, hc = _ssd(orc, p, chunk=chunk)
    assert _rel(yc, y) < 1e-12
    assert _rel(hc, hf) < 1e-12


def test_ssd_p1_equals_m1_constant_a(orc):
    """An SSD head with P = 1 is a Mamba-1 channel whose A is the same for
    every state."""
    p = ssd_problem(13, 2, 30, 1, 1, 16, G=1, gs=4, gate=True, h0=True)
    y, hf = _ssd(orc, p)
    A1 = np.full((1, 16), p["A"][0], np.float32)
    m = dict(x=p["x"].transpose(0, 2, 3, 1).reshape(2, 1, 30), dt=p["dt"].transpose(0, 2, 1),
             z=p["z"].transpose(0, 2, 3, 1).reshape(2, 1, 30), B=p["B"].transpose(0, 2, 3, 1),
             C=p["C"].transpose(0, 2, 3, 1))
    ym, hm = orc.m1_scan(m["x"], m["dt"], A1, m["B"], m["C"], p["B_scale"], p["C_scale"], 4,
                         x_group=p["x_group"][:1], x_scale=p["x_scale"], D=p["D"], z=m["z"],
                         h0=p["h0"].reshape(2, 1, 16))
    assert _rel(ym.reshape(2, 30), y.reshape(2, 30)) < 1e-13
    assert _rel(hm.reshape(2, 16), hf.reshape(2, 16)) < 1e-13


def test_ssd_delta_zero(orc):
    p = ssd_problem(14, 1, 20, 2, 4, 8, gs=4, h0=True)
    p["dt"][:] = 0
    y, hf = _ssd(orc, p, dt_softplus=False)
    np.testing.assert_array_equal(hf.reshape(p["h0"].shape), p["h0"].astype(np.float64))
    yd, _ = ssd_dual(p, softplus=False)
    assert _rel(y.reshape(yd.shape), yd) < 1e-13


# ---- decode ---------------------------------------------------------------------

def test_decode_chain_equals_ssd_scan(orc):
    """L single-token steps from h0 reproduce the SSD scan's y and state."""
    p = ssd_problem(21, 2, 12, 4, 8, 16, G=2, gs=4, gate=True, h0=True, bias=True)
    y, hf = _ssd(orc, p)
    state = p["h0"].astype(np.float64).reshape(8, 8, 16).copy()
    for t in range(12):
        yt = orc.decode_step(state, p["x"][:, t], p["dt"][:, t], p["A"], p["B"][:, t], p["C"][:, t],
                             p["B_scale"], p["C_scale"], 4, x_group=p["x_group"],
                             x_scale=p["x_scale"], D=p["D"], z=p["z"][:, t],
                             dt_bias=p["dt_bias"])
        assert _rel(yt, y.reshape(8, 12, 8)[:, t, :]) < 1e-13
    assert _rel(state, hf.reshape(8, 8, 16)) < 1e-13


def test_decode_from_zero_closed_form(orc):
    """From h = 0 one step gives h = delta x_p B_n (outer product) and
    y = C . h + D x."""
    p = ssd_problem(22, 3, 1, 4, 8, 16, G=1, gs=8)
    state = np.zeros((12, 8, 16))
    y = orc.decode_step(state, p["x"][:, 0], p["dt"][:, 0], p["A"], p["B"][:, 0], p["C"][:, 0],
                        p["B_scale"], p["C_scale"], 8, x_group=p["x_group"], x_scale=p["x_scale"],
                        D=p["D"])
    dl = np.logaddexp(0.0, p["dt"][:, 0].astype(np.float64))  # (b, H)
    x = p["x"][:, 0].astype(np.float64) * p["x_scale"][p["x_group"]].reshape(1, 4, 8)
    Bv = _deq_bc(p["B"][:, 0], p["B_scale"], 8, 2)[:, 0]  # (b, N)
    Cv = _deq_bc(p["C"][:, 0], p["C_scale"], 8, 2)[:, 0]
    h = dl[:, :, None, None] * x[:, :, :, None] * Bv[:, None, None, :]
    assert _rel(state.reshape(h.shape), h) < 1e-14
    want = np.einsum("bhpn,bn->bhp", h, Cv) + p["D"][None, :, None] * x
    assert _rel(y.reshape(want.shape), want) < 1e-14


def test_m1_decode_chain_equals_m1_scan(orc):
    p = m1_problem(23, 2, 10, 6, 16, G=2, gs=4, gate=True, h0=True, bias=True)
    y, hf = _m1(orc, p)
    state = p["h0"].astype(np.float64).reshape(12, 16).copy()
    for t in range(10):
        yt = orc.m1_decode_step(state, p["x"][:, :, t], p["dt"][:, :, t], p["A"],
                                p["B"][:, :, :, t], p["C"][:, :, :, t], p["B_scale"],
                                p["C_scale"], 4, x_group=p["x_group"], x_scale=p["x_scale"],
                                D=p["D"], z=p["z"][:, :, t], dt_bias=p["dt_bias"])
        assert _rel(yt, y[:, t]) < 1e-13
    assert _rel(state, hf) < 1e-13
