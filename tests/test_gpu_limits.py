"""Size limits on the GPU: the 64-bit index path of the streaming kernels
(more than 2^32 elements, ragged end) and very long sequences for both scans,
each against the oracle on sampled outputs (the oracle computes them one by
one; the full outputs are too large for it)."""
import numpy as np
import pytest
import torch

from gpu_util import H, T, assert_scan_close, dev
from problems import m1_problem, oracle_kwargs, ssd_problem
from quantized_state_space_b200 import api

pytestmark = pytest.mark.gpu

BIG = (1 << 32) + 4096 + 3  # elements: past 2^32, not a multiple of 16


@pytest.fixture(scope="module")
def big_x():
    g = torch.Generator(device=dev())
    g.manual_seed(1234)
    x = torch.randn(BIG, dtype=torch.float16, device=dev(), generator=g)
    yield x
    del x
    torch.cuda.empty_cache()


def _sample_idx(rng):
    idx = np.concatenate([rng.integers(0, BIG, size=200_000),
                          np.arange(BIG - 64, BIG), np.arange(0, 64),
                          np.arange((1 << 32) - 32, (1 << 32) + 32)])
    return np.unique(idx)


def test_quantize_past_2_to_32_elements(orc, big_x):
    """outer 1, mid 1, inner BIG: the general path with 64-bit indices."""
    s = np.array([np.float32(3.0 / 127)], np.float32)
    q = torch.empty(BIG, dtype=torch.int8, device=big_x.device)
    api.quantize_groups(big_x, 1, 1, BIG, T(np.zeros(1, np.int32)), 1, scales=T(s), out=q)
    torch.cuda.synchronize()
    idx = _sample_idx(np.random.default_rng(5))
    it = torch.as_tensor(idx, device=big_x.device)
    xs = H(big_x[it])
    got = H(q[it])
    ref, _, _ = orc.quantize_groups(xs, 1, 1, xs.size, np.zeros(1, np.int32), 1,
                                    orc.SCALE_STATIC, s)
    np.testing.assert_array_equal(got, ref)
    del q


def test_softedge_encode_past_2_to_32_elements(orc, big_x):
    s, lo, hi = np.float32(3.5 / 63), 0.06, 3.5
    codes = api.softedge_encode(big_x, s, lo, hi, 2)
    torch.cuda.synchronize()
    idx = _sample_idx(np.random.default_rng(6))
    it = torch.as_tensor(idx, device=big_x.device)
    xs = H(big_x[it])
    ref, _ = orc.softedge_encode(xs, s, lo, hi, 2)
    np.testing.assert_array_equal(H(codes[it]), ref)
    del codes


@pytest.mark.parametrize("L", [(1 << 20) + 16, (1 << 20) + 5])
def test_scan_million_step_sequence(orc, L):
    """A million-step Mamba-1 sequence (16-byte rows and ragged rows); four
    channels of each batch row are recomputed by the oracle."""
    b, d, N_ = 2, 32, 16
    p = m1_problem(950, b, L, d, N_, gate=True, h0=True, bias=True)
    y, hf = api.selective_scan(T(p["x"]), T(p["dt"]), T(p["A"]), T(p["B"]), T(p["C"]),
                               T(p["B_scale"]), T(p["C_scale"]), p["state_group_size"],
                               x_group=T(p["x_group"]), x_scale=T(p["x_scale"]), D=T(p["D"]),
                               z=T(p["z"]), dt_bias=T(p["dt_bias"]), h0=T(p["h0"]))
    units = np.array([0, 13, 31, d + 7], dtype=np.int64)  # (batch, channel) pairs b * d + c
    yo, ho = orc.m1_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["B_scale"], p["C_scale"],
                         p["state_group_size"], units=units, **oracle_kwargs(p))
    yg = H(y).reshape(b * d, L)[units].astype(np.float64)
    hg = H(hf).reshape(b * d, N_)[units]
    assert_scan_close(yg, yo, hg, ho)


def test_ssd_long_sequence(orc):
    """A 65 553-step SSD sequence (ragged last tile); every head recomputed."""
    b, L, Hh, P, N_ = 1, 65536 + 17, 2, 64, 128
    p = ssd_problem(960, b, L, Hh, P, N_, G=1, gs=8, gate=True, h0=True)
    y, hf = api.ssd_chunk_scan(T(p["x"]), T(p["dt"]), T(p["A"]), T(p["B"]), T(p["C"]),
                               T(p["B_scale"]), T(p["C_scale"]), 8, x_group=T(p["x_group"]),
                               x_scale=T(p["x_scale"]), D=T(p["D"]), z=T(p["z"]), h0=T(p["h0"]))
    yo, ho = orc.ssd_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["B_scale"], p["C_scale"], 8,
                          **oracle_kwargs(p))
    yg = np.moveaxis(H(y).astype(np.float64), 2, 1).reshape(b * Hh, L, P)
    assert_scan_close(yg, yo.reshape(yg.shape), H(hf), ho.reshape(H(hf).shape))
