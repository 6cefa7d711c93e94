"""GPU Mamba-2 SSD chunked scan (tcgen05) vs the oracle (SSDi8 abstract;
Quamba2 abstract: W8A8 Mamba2 backbone).

Tolerances: max |y - y_ref| <= 2e-3 max |y_ref|, final state rel-L2 <= 1e-4."""
import numpy as np
import pytest
import torch

from gpu_util import H, T, assert_scan_close, dev, status_word, y_err, state_err
from problems import oracle_kwargs, ssd_problem
from quantized_state_space_b200 import _native as N
from quantized_state_space_b200 import api, calibrate, synth

pytestmark = pytest.mark.gpu


def gpu_ssd(p, chunk=256, **kw):
    args = dict(D=T(p["D"]), z=T(p["z"]), dt_bias=T(p["dt_bias"]), h0=T(p.get("h0")))
    if p["x"].dtype == np.uint8:
        args["se_scale"] = p["se_scale"]
    else:
        args["x_group"] = T(p["x_group"])
        args["x_scale"] = T(p["x_scale"])
    args.update(kw)
    y, hf = api.ssd_chunk_scan(T(p["x"]), T(p["dt"]), T(p["A"]), T(p["B"]), T(p["C"]),
                               T(p["B_scale"]), T(p["C_scale"]), p["state_group_size"],
                               chunk=chunk, **args)
    return H(y).astype(np.float64), H(hf)


def oracle_ssd(orc, p, **kw):
    return orc.ssd_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["B_scale"], p["C_scale"],
                        p["state_group_size"], **oracle_kwargs(p), **kw)


CASES = [
    # (b, L, H, G, gs, gate, h0, bias, fmt, dt_mean)
    (1, 128, 2, 1, 8, False, False, False, "int8", -4.0),   # one tile
    (2, 300, 3, 1, 8, True, True, True, "int8", -4.0),      # ragged last tile, h0, gate
    (1, 64, 4, 2, 4, False, True, False, "int8", -4.0),     # shorter than a tile, G = 2
    (1, 1, 2, 1, 8, False, True, False, "int8", -4.0),      # one step
    (2, 512, 4, 4, 16, True, False, True, "int8", -2.0),    # strong decay, G = 4
    (1, 384, 2, 1, 8, True, True, False, "softedge", -4.0),
    (1, 1000, 2, 1, 8, False, False, False, "int8", -5.0),  # weak decay, long
]


@pytest.mark.parametrize("ci", range(len(CASES)))
def test_ssd_vs_oracle(orc, ci):
    b, L, Hh, G, gs, gate, h0, bias, fmt, dtm = CASES[ci]
    p = ssd_problem(400 + ci, b, L, Hh, 64, 128, G=G, gs=gs, gate=gate, h0=h0, bias=bias,
                    x_format=fmt, dt_mean=dtm)
    st = status_word()
    y, hf = gpu_ssd(p, status=st)
    yo, ho = oracle_ssd(orc, p)
    assert int(H(st)[0]) == 0
    assert_scan_close(y.transpose(0, 2, 1, 3).reshape(yo.shape), yo, hf.reshape(ho.shape), ho)


@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_ssd_chunk_lengths_agree(orc, chunk):
    p = ssd_problem(450, 1, 520, 2, 64, 128, gate=True, h0=True)
    y, hf = gpu_ssd(p, chunk=chunk)
    yo, ho = oracle_ssd(orc, p)
    assert_scan_close(y.transpose(0, 2, 1, 3).reshape(yo.shape), yo, hf.reshape(ho.shape), ho)


def test_ssd_split_with_state_bit_exact():
    """One pass per sequence (max_segments = 1): scan(L) equals scan(first 256
    steps) then scan(rest, h0 = its state), byte for byte."""
    p = ssd_problem(460, 2, 512, 2, 64, 128, gate=True)
    y, hf = gpu_ssd(p, max_segments=1)
    a, b = dict(p), dict(p)
    for k in ("x", "dt", "z", "B", "C"):
        a[k] = np.ascontiguousarray(p[k][:, :256])
        b[k] = np.ascontiguousarray(p[k][:, 256:])
    ya, ha = gpu_ssd(a, max_segments=1)
    b["h0"] = ha
    yb, hb = gpu_ssd(b, max_segments=1)
    np.testing.assert_array_equal(np.concatenate([ya, yb], axis=1), y)
    np.testing.assert_array_equal(hb, hf)


SEG_CASES = [
    # (b, L, H, G, gate, h0, max_segments, units checked (None: all))
    (1, 128 * 40 + 37, 2, 1, True, True, 0, None),    # 2 sequences, 21 segments, ragged end
    (1, 128 * 9, 3, 1, False, True, 4, None),         # at most 4 segments: 3 of 3 tiles
    (1, 128 * 3 + 1, 1, 1, True, True, 0, None),      # last segment a single step
    (2, 1024, 80, 4, True, False, 0,                  # 160 sequences: whole ones and cut ones
     [0, 1, 77, 100, 147, 148, 150, 155, 159]),
    (1, 128 * 7 + 3, 2, 1, True, True, 0, None, "softedge"),  # soft-edge x codes, cut
    (2, 512, 74, 2, False, True, 0, [0, 73, 74, 147]),  # 148 sequences: one full round, no cut
    (1, 128 * 6, 2, 1, True, True, 64, None),         # max_segments above the plan's cap
]


@pytest.mark.parametrize("ci", range(len(SEG_CASES)))
def test_ssd_segments_vs_oracle(orc, ci):
    """Sequences cut into segments (the segment start states carried by the
    second kernel) against the oracle, and against one pass per sequence."""
    b, L, Hh, G, gate, h0, ms, units = SEG_CASES[ci][:8]
    fmt = SEG_CASES[ci][8] if len(SEG_CASES[ci]) > 8 else "int8"
    p = ssd_problem(490 + ci, b, L, Hh, 64, 128, G=G, gate=gate, h0=h0, bias=True, x_format=fmt)
    st = status_word()
    y, hf = gpu_ssd(p, max_segments=ms, status=st)
    assert int(H(st)[0]) == 0
    u = np.arange(b * Hh) if units is None else np.asarray(units, np.int64)
    yo, ho = orc.ssd_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["B_scale"], p["C_scale"],
                          p["state_group_size"], units=None if units is None else u,
                          **oracle_kwargs(p))
    yg = y.transpose(0, 2, 1, 3).reshape(b * Hh, L, 64)[u]
    hg = hf.reshape(b * Hh, 64, 128)[u]
    assert_scan_close(yg, yo.reshape(yg.shape), hg, ho.reshape(hg.shape))
    y1, h1 = gpu_ssd(p, max_segments=1)
    assert_scan_close(y, y1, hf, h1)


def test_ssd_delta_zero(orc):
    p = ssd_problem(470, 1, 200, 2, 64, 128, h0=True)
    p["dt"][:] = 0
    y, hf = gpu_ssd(p, dt_softplus=False)
    yo, ho = oracle_ssd(orc, p, dt_softplus=False)
    assert_scan_close(y.transpose(0, 2, 1, 3).reshape(yo.shape), yo, hf.reshape(ho.shape), ho)
    np.testing.assert_allclose(hf, p["h0"], rtol=0, atol=0)


@pytest.mark.parametrize("max_segments", [0, 1])
def test_ssd_head_permutation_bit_exact(max_segments):
    """Quamba2 compute invariance for the SSD form: permuting the heads with
    their x cluster ids, dt, z, A, D, dt_bias and h0 permutes y and the final
    state exactly (with segments on, all 12 sequences share one SM round and
    are cut alike)."""
    Hh, P = 6, 64
    p = ssd_problem(950, 2, 300, Hh, P, 128, gate=True, h0=True, bias=True)
    perm = np.random.default_rng(2).permutation(Hh)
    q = dict(p)
    for k in ("x", "dt", "z"):
        q[k] = np.ascontiguousarray(p[k][:, :, perm])
    q["x_group"] = np.ascontiguousarray(p["x_group"].reshape(Hh, P)[perm].reshape(-1))
    for k in ("A", "D", "dt_bias"):
        q[k] = np.ascontiguousarray(p[k][perm])
    q["h0"] = np.ascontiguousarray(p["h0"][:, perm])
    y, hf = gpu_ssd(p, max_segments=max_segments)
    yq, hq = gpu_ssd(q, max_segments=max_segments)
    np.testing.assert_array_equal(yq, y[:, :, perm])
    np.testing.assert_array_equal(hq, hf[:, perm])


def test_ssd_bad_group_status():
    p = ssd_problem(480, 1, 128, 2, 64, 128)
    p["x_group"][5] = 1000
    st = status_word()
    gpu_ssd(p, status=st)
    assert int(H(st)[0]) & N.DEV_BAD_GROUP


def test_ssd27b_workload_end_to_end(orc):
    """The Mamba-2-2.7B-shaped SSD layer (b 4, L 4096, H 80, P 64, N 128, G 1)
    from raw activations: host calibration, GPU quantizers, GPU SSD; the
    oracle repeats every step from the raw arrays on sampled heads."""
    dm, raw = synth.workload_inputs("ssd27b")
    b, L, Hh, P, Nst, G, gs, k = (dm["batch"], dm["seqlen"], dm["nheads"], dm["headdim"],
                                  dm["dstate"], dm["ngroups"], dm["state_group_size"],
                                  dm["x_clusters"])
    grp, xs = calibrate.ssd_x_clusters(raw["x"], k)
    smap = calibrate.state_group_map(G, Nst, gs)
    bs = calibrate.state_group_absmax_scales(raw["B"], G, Nst, gs, "lgn")
    cs = calibrate.state_group_absmax_scales(raw["C"], G, Nst, gs, "lgn")
    xq, _ = api.quantize_groups(T(raw["x"]), b * L, Hh * P, 1, T(grp), k, scales=T(xs))
    Bq, _ = api.quantize_groups(T(raw["B"]), b * L, G * Nst, 1, T(smap), G * Nst // gs, scales=T(bs))
    Cq, _ = api.quantize_groups(T(raw["C"]), b * L, G * Nst, 1, T(smap), G * Nst // gs, scales=T(cs))
    st = status_word()
    y, hf = api.ssd_chunk_scan(xq, T(raw["dt"]), T(raw["A"]), Bq, Cq, T(bs), T(cs), gs,
                               chunk=dm["chunk"], x_group=T(grp), x_scale=T(xs), D=T(raw["D"]),
                               status=st)
    torch.cuda.synchronize()
    assert int(H(st)[0]) == 0
    # oracle chain
    head_abs = np.abs(raw["x"].astype(np.float32)).max(axis=(0, 1, 3))
    ohc, oxs = orc.cluster_by_absmax(head_abs.astype(np.float64), k)
    ogrp = np.repeat(ohc, P).astype(np.int32)
    omap = np.arange(G * Nst) // gs
    _, obs, _ = orc.quantize_groups(raw["B"], b * L, G * Nst, 1, omap, G * Nst // gs, orc.SCALE_ABSMAX)
    _, ocs, _ = orc.quantize_groups(raw["C"], b * L, G * Nst, 1, omap, G * Nst // gs, orc.SCALE_ABSMAX)
    ox, _, _ = orc.quantize_groups(raw["x"], b * L, Hh * P, 1, ogrp, k, orc.SCALE_STATIC, oxs)
    oB, _, _ = orc.quantize_groups(raw["B"], b * L, G * Nst, 1, omap, G * Nst // gs, orc.SCALE_STATIC, obs)
    oC, _, _ = orc.quantize_groups(raw["C"], b * L, G * Nst, 1, omap, G * Nst // gs, orc.SCALE_STATIC, ocs)
    np.testing.assert_array_equal(H(xq), ox)
    np.testing.assert_array_equal(H(Bq), oB)
    # sampled heads, including the fastest- and slowest-decaying ones
    rng = np.random.default_rng(2)
    units = set(rng.choice(b * Hh, size=6, replace=False).tolist())
    units |= {int(np.argmin(raw["A"])), int(np.argmax(raw["A"])) + Hh}
    units = np.array(sorted(units))
    yo, ho = orc.ssd_scan(ox, raw["dt"], raw["A"], oB, oC, obs, ocs, gs, x_group=ogrp,
                          x_scale=oxs, D=raw["D"], units=units)
    yg = H(y).astype(np.float64)  # (b, L, H, P)
    yg = np.stack([yg[u // Hh, :, u % Hh, :] for u in units])
    hg = H(hf).reshape(b * Hh, P, Nst)[units]
    assert_scan_close(yg, yo, hg, ho)


def test_ssd_int8_y_bit_exact():
    """Persistent-INT8 epilogue (SSDi8 abstract): int8 y whose bytes equal the
    quantizer applied to the binary16 y; with the binary16 y dropped the codes
    and the state are unchanged."""
    b, L, Hh, P, N_ = 2, 384, 4, 64, 128
    p = ssd_problem(860, b, L, Hh, P, N_, G=1, gs=8, gate=True, h0=True)
    rng = np.random.default_rng(861)
    ky = 6
    ygrp = rng.integers(0, ky, size=Hh * P).astype(np.int32)
    ysc = synth.random_scales(rng, ky, 0.002, 0.02)
    kw = dict(x_group=T(p["x_group"]), x_scale=T(p["x_scale"]), D=T(p["D"]), z=T(p["z"]),
              h0=T(p["h0"]), y_group=T(ygrp), y_scale=T(ysc))
    args = (T(p["x"]), T(p["dt"]), T(p["A"]), T(p["B"]), T(p["C"]), T(p["B_scale"]),
            T(p["C_scale"]), 8)
    y, hf, yq = api.ssd_chunk_scan(*args, **kw)
    ref, _ = api.quantize_groups(y, b * L, Hh * P, 1, T(ygrp), ky, scales=T(ysc))
    np.testing.assert_array_equal(H(yq), H(ref))
    y2, hf2, yq2 = api.ssd_chunk_scan(*args, want_y=False, **kw)
    assert y2 is None
    np.testing.assert_array_equal(H(yq2), H(yq))
    np.testing.assert_array_equal(H(hf2).view(np.uint32), H(hf).view(np.uint32))


@pytest.mark.parametrize("cuts", [(0, 512), (0, 384, 768, 1000), (0, 127, 128, 900)])
def test_ssd_sequence_sharded_vs_oracle(orc, cuts):
    """Sequence sharding emulated in one process: each slice scanned from a
    zero state (the first from h0) with its total decay, the summaries folded
    by the state-chain kernel, each later slice's carried start state added
    by the carry-in kernel; the concatenated y and the folded final state
    against the oracle's unsplit scan."""
    b, L, Hh = 2, 1100, 3
    p = ssd_problem(940, b, L, Hh, 64, 128, G=1, gate=True, h0=True, bias=True)
    yo, ho = oracle_ssd(orc, p)
    bounds = list(cuts) + [L]
    ys, h_ends, decs = [], [], []
    for r in range(len(bounds) - 1):
        sl = slice(bounds[r], bounds[r + 1])
        q = dict(p)
        for k in ("x", "dt", "z", "B", "C"):
            q[k] = np.ascontiguousarray(p[k][:, sl])
        args = (T(q["x"]), T(q["dt"]), T(q["A"]), T(q["B"]), T(q["C"]), T(q["B_scale"]),
                T(q["C_scale"]), 8)
        kw = dict(x_group=T(q["x_group"]), x_scale=T(q["x_scale"]), D=T(q["D"]), z=T(q["z"]),
                  dt_bias=T(q["dt_bias"]))
        dec = torch.empty((b, Hh), dtype=torch.float32, device=dev())
        y, he = api.ssd_chunk_scan(*args, h0=T(p["h0"]) if r == 0 else None, dec_final=dec,
                                   **kw)
        # the total decay: sum_t delta_t A_h log2(e)
        dt = q["dt"].astype(np.float64) + q["dt_bias"].astype(np.float64)
        ref = (np.logaddexp(0.0, dt) * q["A"].astype(np.float64)).sum(axis=1) * np.log2(np.e)
        np.testing.assert_allclose(H(dec), ref, rtol=2e-5, atol=1e-4)
        if r > 0:
            carry = api.state_chain(h_ends, decs)
            api.ssd_carry_in(*args, carry, y, **kw)
        ys.append(H(y).astype(np.float64))
        h_ends.append(he)
        decs.append(dec)
    hf = H(api.state_chain(h_ends, decs))
    y = np.concatenate(ys, axis=1)
    assert_scan_close(y.transpose(0, 2, 1, 3).reshape(yo.shape), yo, hf.reshape(ho.shape), ho)


def test_ssd_carry_in_h_final_and_dec_with_segments(orc):
    """dec_final of sequences cut into segments (the second kernel sums the
    segments' decays) and the carry-in's h_final update, on one call."""
    b, L, Hh = 1, 128 * 9 + 5, 2
    p = ssd_problem(950, b, L, Hh, 64, 128, gate=False, h0=False, bias=True)
    args = (T(p["x"]), T(p["dt"]), T(p["A"]), T(p["B"]), T(p["C"]), T(p["B_scale"]),
            T(p["C_scale"]), 8)
    kw = dict(x_group=T(p["x_group"]), x_scale=T(p["x_scale"]), D=T(p["D"]),
              dt_bias=T(p["dt_bias"]))
    dec = torch.empty((b, Hh), dtype=torch.float32, device=dev())
    y, hf = api.ssd_chunk_scan(*args, dec_final=dec, **kw)  # two sequences: cut
    dt = p["dt"].astype(np.float64) + p["dt_bias"].astype(np.float64)
    ref = (np.logaddexp(0.0, dt) * p["A"].astype(np.float64)).sum(axis=1) * np.log2(np.e)
    np.testing.assert_allclose(H(dec), ref, rtol=2e-5, atol=1e-4)
    rng = np.random.default_rng(951)
    h_start = (rng.standard_normal((b, Hh, 64, 128)) * 0.1).astype(np.float32)
    api.ssd_carry_in(*args, T(h_start), y, h_final=hf, **kw)
    q = dict(p)
    q["h0"] = h_start
    yo, ho = oracle_ssd(orc, q)
    assert_scan_close(H(y).astype(np.float64).transpose(0, 2, 1, 3).reshape(yo.shape), yo,
                      H(hf).reshape(ho.shape), ho)


def test_state_chain_and_carry_in_edge_cases():
    """A one-part fold is the part itself; a three-part fold matches numpy;
    carry-in on an empty sequence adds h_carry to h_final and nothing else."""
    rng = np.random.default_rng(960)
    he = rng.standard_normal((3, 2, 5, 4, 8)).astype(np.float32)
    dc = -rng.uniform(0.0, 3.0, size=(3, 2, 5)).astype(np.float32)
    np.testing.assert_array_equal(H(api.state_chain([T(he[0])], [T(dc[0])])), he[0])
    ref = np.zeros(he.shape[1:], np.float64)
    for q in range(3):
        ref = np.exp2(dc[q].astype(np.float64))[..., None, None] * ref + he[q]
    np.testing.assert_allclose(H(api.state_chain(T(he), T(dc))), ref, rtol=1e-5, atol=1e-6)
    p = ssd_problem(961, 1, 0, 2, 64, 128)
    hf = (rng.standard_normal((1, 2, 64, 128)) * 0.1).astype(np.float32)
    hc = (rng.standard_normal((1, 2, 64, 128)) * 0.1).astype(np.float32)
    args = (T(p["x"]), T(p["dt"]), T(p["A"]), T(p["B"]), T(p["C"]), T(p["B_scale"]),
            T(p["C_scale"]), 8)
    y = torch.empty((1, 0, 2, 64), dtype=torch.float16, device=dev())
    hft = T(hf)
    api.ssd_carry_in(*args, T(hc), y, x_group=T(p["x_group"]), x_scale=T(p["x_scale"]),
                     h_final=hft)
    np.testing.assert_array_equal(H(hft), hf + hc)


# ---- the pipelined kernel against the single-schedule kernel ---------------
# SSMQ_SSD_KERNEL=pipelined selects, for binary16 y, a kernel whose warp roles
# work on different tiles at once; it keeps the default kernel's arithmetic
# operation for operation, so the two give the same bits.

PIPE_CASES = [
    # (b, L, H, G, gs, gate, h0, bias, fmt, dt_mean, max_segments)
    (1, 128, 2, 1, 8, False, False, False, "int8", -4.0, 1),
    (2, 300, 3, 1, 8, True, True, True, "int8", -4.0, 0),
    (1, 1, 2, 1, 8, False, True, False, "int8", -4.0, 0),
    (2, 512, 4, 4, 16, True, False, True, "int8", -2.0, 0),
    (1, 384, 2, 1, 8, True, True, False, "softedge", -4.0, 0),
    (1, 1000, 2, 1, 8, False, False, False, "int8", -5.0, 1),
    (2, 2048, 5, 1, 8, False, True, True, "int8", -4.0, 0),   # segments of the last round
    (1, 640, 2, 2, 8, False, False, False, "int8", 0.5, 1),   # very strong decay: per-element branch
]


@pytest.mark.parametrize("ci", range(len(PIPE_CASES)))
def test_ssd_pipelined_equals_single_schedule(ci, monkeypatch):
    b, L, Hh, G, gs, gate, h0, bias, fmt, dtm, ms = PIPE_CASES[ci]
    p = ssd_problem(470 + ci, b, L, Hh, 64, 128, G=G, gs=gs, gate=gate, h0=h0, bias=bias,
                    x_format=fmt, dt_mean=dtm)
    dec_a = torch.zeros((b, Hh), dtype=torch.float32, device=dev())
    dec_b = torch.zeros((b, Hh), dtype=torch.float32, device=dev())
    st_a, st_b = status_word(), status_word()
    monkeypatch.setenv("SSMQ_SSD_KERNEL", "pipelined")
    ya, ha = gpu_ssd(p, max_segments=ms, dec_final=dec_a, status=st_a)
    monkeypatch.delenv("SSMQ_SSD_KERNEL")
    yb, hb = gpu_ssd(p, max_segments=ms, dec_final=dec_b, status=st_b)
    torch.cuda.synchronize()
    assert int(H(st_a)[0]) == 0 and int(H(st_b)[0]) == 0
    np.testing.assert_array_equal(ya.astype(np.float16).view(np.uint16),
                                  yb.astype(np.float16).view(np.uint16))
    np.testing.assert_array_equal(ha.view(np.uint32), hb.view(np.uint32))
    np.testing.assert_array_equal(H(dec_a).view(np.uint32), H(dec_b).view(np.uint32))
