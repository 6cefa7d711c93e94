"""GPU single-token decode state update vs the oracle (Quamba2 abstract:
generation stage of W8A8 Mamba2 models)."""
import numpy as np
import pytest
import torch

from gpu_util import H, T, assert_scan_close, dev, state_err, y_err, STATE_TOL, Y_TOL
from problems import ssd_problem
from quantized_state_space_b200 import api, calibrate, synth

pytestmark = pytest.mark.gpu

CASES = [
    # (b, H, P, N, G, gs, gate, bias, fmt)
    (3, 8, 64, 128, 2, 8, False, False, "int8"),
    (2, 6, 40, 64, 3, 4, True, True, "int8"),     # ragged P
    (4, 4, 17, 32, 1, 8, True, False, "int8"),
    (2, 4, 64, 16, 4, 4, False, True, "int8"),
    (2, 8, 64, 128, 8, 8, True, False, "softedge"),
    (1, 1, 1, 16, 1, 16, False, False, "int8"),
]


@pytest.mark.parametrize("ci", range(len(CASES)))
def test_decode_chain_vs_oracle(orc, ci):
    b, Hh, P, N_, G, gs, gate, bias, fmt = CASES[ci]
    steps = 24
    p = ssd_problem(200 + ci, b, steps, Hh, P, N_, G=G, gs=gs, gate=gate, bias=bias, h0=True,
                    x_format=fmt)
    state = T(p["h0"])
    ref = p["h0"].astype(np.float64).reshape(b * Hh, P, N_).copy()
    kw = dict(D=T(p["D"]), dt_bias=T(p["dt_bias"]))
    okw = dict(D=p["D"], dt_bias=p["dt_bias"])
    if fmt == "softedge":
        kw["se_scale"] = okw["se_scale"] = p["se_scale"]
    else:
        kw.update(x_group=T(p["x_group"]), x_scale=T(p["x_scale"]))
        okw.update(x_group=p["x_group"], x_scale=p["x_scale"])
    for t in range(steps):
        xt = np.ascontiguousarray(p["x"][:, t])
        zt = None if p["z"] is None else np.ascontiguousarray(p["z"][:, t])
        y = api.state_update(state, T(xt), T(np.ascontiguousarray(p["dt"][:, t])), T(p["A"]),
                             T(np.ascontiguousarray(p["B"][:, t])),
                             T(np.ascontiguousarray(p["C"][:, t])), T(p["B_scale"]),
                             T(p["C_scale"]), gs, z=T(zt), **kw)
        yo = orc.decode_step(ref, xt, p["dt"][:, t], p["A"], p["B"][:, t], p["C"][:, t],
                             p["B_scale"], p["C_scale"], gs, z=zt, **okw)
        assert y_err(H(y).reshape(yo.shape), yo) <= Y_TOL
    assert state_err(H(state).reshape(ref.shape), ref) <= STATE_TOL


def _decode_workload(steps):
    dm, raw = synth.workload_inputs("decode8b", steps=steps)
    return dm, raw


def test_decode8b_chain_1000_steps(orc):
    """The Mamba-2-8B-shaped decode (b 64, H 128, P 64, N 128, G 8) for 1000
    chained steps; y of every step and the final state are compared on a
    sample of (batch, head) pairs."""
    dm, raw = _decode_workload(1000)
    b, Hh, P, N_, G, gs, S = (dm["batch"], dm["nheads"], dm["headdim"], dm["dstate"],
                              dm["ngroups"], dm["state_group_size"], dm["steps"])
    k = dm["x_clusters"]
    # product: offline calibration, GPU quantization of all steps, GPU chain
    grp, xs = calibrate.ssd_x_clusters(raw["x"], k)
    bs = calibrate.state_group_absmax_scales(raw["B"], G, N_, gs, "gn")
    cs = calibrate.state_group_absmax_scales(raw["C"], G, N_, gs, "gn")
    smap = np.arange(G * N_) // gs
    xq, _ = api.quantize_groups(T(raw["x"]), S * b, Hh * P, 1, T(grp), k, scales=T(xs))
    Bq, _ = api.quantize_groups(T(raw["B"]), S * b, G * N_, 1, T(smap.astype(np.int32)),
                                G * N_ // gs, scales=T(bs))
    Cq, _ = api.quantize_groups(T(raw["C"]), S * b, G * N_, 1, T(smap.astype(np.int32)),
                                G * N_ // gs, scales=T(cs))
    dt = T(raw["dt"])
    state = T(raw["state"])
    A, D, grp_t, xs_t, bs_t, cs_t = T(raw["A"]), T(raw["D"]), T(grp), T(xs), T(bs), T(cs)
    rng = np.random.default_rng(1)
    units = np.sort(rng.choice(b * Hh, size=12, replace=False))
    ys = []
    for t in range(S):
        y = api.state_update(state, xq[t], dt[t], A, Bq[t], Cq[t], bs_t, cs_t, gs, x_group=grp_t,
                             x_scale=xs_t, D=D)
        ys.append(y.view(b * Hh, P)[torch.as_tensor(units, device=dev())].clone())
    torch.cuda.synchronize()
    yg = np.stack([H(v) for v in ys]).astype(np.float64)  # (S, units, P)
    # oracle: own calibration + quantizers on the sampled heads' inputs
    head_abs = np.abs(raw["x"].astype(np.float32)).reshape(-1, Hh, P).max(axis=(0, 2))
    ohc, oxs = orc.cluster_by_absmax(head_abs.astype(np.float64), k)
    ogrp = np.repeat(ohc, P).astype(np.int32)
    np.testing.assert_array_equal(ogrp, grp)
    _, obs, _ = orc.quantize_groups(raw["B"], S * b, G * N_, 1, smap, G * N_ // gs, orc.SCALE_ABSMAX)
    _, ocs, _ = orc.quantize_groups(raw["C"], S * b, G * N_, 1, smap, G * N_ // gs, orc.SCALE_ABSMAX)
    ref = raw["state"].astype(np.float64).reshape(b * Hh, P, N_)[units].copy()
    yo = np.zeros((S, units.size, P))
    for t in range(S):
        ox, _, _ = orc.quantize_groups(raw["x"][t], b, Hh * P, 1, ogrp, k, orc.SCALE_STATIC, oxs)
        oB, _, _ = orc.quantize_groups(raw["B"][t], b, G * N_, 1, smap, G * N_ // gs,
                                       orc.SCALE_STATIC, obs)
        oC, _, _ = orc.quantize_groups(raw["C"][t], b, G * N_, 1, smap, G * N_ // gs,
                                       orc.SCALE_STATIC, ocs)
        if t == 0:
            np.testing.assert_array_equal(H(xq[0]), ox)
        yo[t] = orc.decode_step(ref, ox, raw["dt"][t], raw["A"], oB, oC, obs, ocs, gs,
                                x_group=ogrp, x_scale=oxs, D=raw["D"], units=units)
    assert y_err(yg, yo) <= Y_TOL
    hf = H(state).reshape(b * Hh, P, N_)[units]
    assert state_err(hf, ref) <= STATE_TOL


def test_decode_checkpoint_resume_bit_exact():
    """1000 steps equal 500 steps, a copy of the state to the host and back,
    and 500 more steps, bit for bit."""
    p = ssd_problem(300, 2, 1000, 4, 64, 128, G=2, gs=8, h0=True)
    kw = dict(x_group=T(p["x_group"]), x_scale=T(p["x_scale"]), D=T(p["D"]))
    X, DT, Bq, Cq = T(p["x"]), T(p["dt"]), T(p["B"]), T(p["C"])
    A, bs, cs = T(p["A"]), T(p["B_scale"]), T(p["C_scale"])

    def run(state, t0, t1):
        for t in range(t0, t1):
            api.state_update(state, X[:, t].contiguous(), DT[:, t].contiguous(), A,
                             Bq[:, t].contiguous(), Cq[:, t].contiguous(), bs, cs, 8, **kw)

    s1 = T(p["h0"])
    run(s1, 0, 1000)
    s2 = T(p["h0"])
    run(s2, 0, 500)
    host = H(s2).copy()
    s3 = T(host)
    run(s3, 500, 1000)
    np.testing.assert_array_equal(H(s3), H(s1))


# ---- Mamba-1 form (A per channel and state) ---------------------------------

from problems import m1_problem  # noqa: E402

M1_CASES = [
    # (b, d, N, G, gs, gate, bias, fmt)
    (3, 64, 16, 1, 4, True, False, "int8"),
    (2, 40, 4, 2, 2, False, True, "int8"),
    (2, 24, 8, 1, 8, True, True, "softedge"),
    (1, 16, 32, 4, 8, False, False, "int8"),
    (2, 8, 64, 1, 16, True, False, "int8"),
    (2, 8, 128, 2, 16, True, True, "int8"),
]


@pytest.mark.parametrize("ci", range(len(M1_CASES)))
def test_m1_decode_chain_vs_oracle(orc, ci):
    b, d, N_, G, gs, gate, bias, fmt = M1_CASES[ci]
    steps = 20
    p = m1_problem(500 + ci, b, steps, d, N_, G=G, gs=gs, gate=gate, h0=True, bias=bias,
                   x_format=fmt)
    state = T(p["h0"])
    ref = p["h0"].astype(np.float64).reshape(b * d, N_).copy()
    kw = dict(D=T(p["D"]), dt_bias=T(p["dt_bias"]))
    okw = dict(D=p["D"], dt_bias=p["dt_bias"])
    if fmt == "softedge":
        kw["se_scale"] = okw["se_scale"] = p["se_scale"]
    else:
        kw.update(x_group=T(p["x_group"]), x_scale=T(p["x_scale"]))
        okw.update(x_group=p["x_group"], x_scale=p["x_scale"])
    for t in range(steps):
        xt = np.ascontiguousarray(p["x"][:, :, t])
        zt = None if p["z"] is None else np.ascontiguousarray(p["z"][:, :, t])
        Bt = np.ascontiguousarray(p["B"][:, :, :, t])
        Ct = np.ascontiguousarray(p["C"][:, :, :, t])
        dtt = np.ascontiguousarray(p["dt"][:, :, t])
        y = api.selective_state_update(state, T(xt), T(dtt), T(p["A"]), T(Bt), T(Ct),
                                       T(p["B_scale"]), T(p["C_scale"]), gs, z=T(zt), **kw)
        yo = orc.m1_decode_step(ref, xt, dtt, p["A"], Bt, Ct, p["B_scale"], p["C_scale"], gs,
                                z=zt, **okw)
        assert y_err(H(y).reshape(yo.shape), yo) <= Y_TOL
    assert state_err(H(state).reshape(ref.shape), ref) <= STATE_TOL


def test_m1_decode_equals_scan_steps():
    """L single-token Mamba-1 steps reproduce the GPU scan's final state."""
    p = m1_problem(520, 2, 64, 32, 16, gate=True, h0=True)
    kw = dict(x_group=T(p["x_group"]), x_scale=T(p["x_scale"]), D=T(p["D"]))
    _, hf = api.selective_scan(T(p["x"]), T(p["dt"]), T(p["A"]), T(p["B"]), T(p["C"]),
                               T(p["B_scale"]), T(p["C_scale"]), 4, z=T(p["z"]), h0=T(p["h0"]),
                               **kw)
    state = T(p["h0"])
    for t in range(64):
        api.selective_state_update(state, T(np.ascontiguousarray(p["x"][:, :, t])),
                                   T(np.ascontiguousarray(p["dt"][:, :, t])), T(p["A"]),
                                   T(np.ascontiguousarray(p["B"][:, :, :, t])),
                                   T(np.ascontiguousarray(p["C"][:, :, :, t])), T(p["B_scale"]),
                                   T(p["C_scale"]), 4, z=T(np.ascontiguousarray(p["z"][:, :, t])),
                                   **kw)
    assert state_err(H(state), H(hf)) <= 1e-5
