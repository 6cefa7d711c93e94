"""Pins of the oracle's quantizers against hand-worked cases, exact rational
arithmetic, numpy's IEEE binary32 division and the codec's invariants.

Quantizer: Quamba-SE write-up (wmrh.cn) section 1; Quamba2 abstract.
Soft-edge codec: Quamba-SE write-up sections 2.1 and 2.2.
"""
from fractions import Fraction

import numpy as np
import pytest

from conftest import golden_rows


def _np_quant(v, s, lim=127):
    """numpy's IEEE binary32 division (correctly rounded) + rint (ties even)."""
    v = np.asarray(v, np.float32)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        r = v / np.float32(s)
    return np.clip(np.rint(r.astype(np.float64)), -lim, lim).astype(np.int64)


# ---- group quantizer --------------------------------------------------------

def test_quantizer_golden(orc):
    for row in golden_rows("quantizer_cases.txt"):
        v, s, want = row.split()
        x = np.array([float(v)], np.float32)
        q, _, _ = orc.quantize_groups(x, 1, 1, 1, [0], 1, orc.SCALE_STATIC,
                                      np.array([float(s)], np.float32))
        assert int(q[0]) == int(want), row


def test_quantizer_matches_numpy_all_f16(orc):
    """Every finite binary16 value, several scales: oracle == numpy fp32 rint."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16)
    vals = vals[np.isfinite(vals)]
    for s in (1.0, 0.0078125, 0.0312345, 3.3e-5, 0.37, 517.0):
        q, _, nf = orc.quantize_groups(vals, 1, 1, vals.size, [0], 1, orc.SCALE_STATIC,
                                       np.array([s], np.float32))
        assert nf == 0
        np.testing.assert_array_equal(q.astype(np.int64), _np_quant(vals.astype(np.float32), s))


def test_quantizer_matches_numpy_random_f32(orc):
    rng = np.random.default_rng(7)
    v = (rng.standard_normal(400_000) * rng.choice([0.01, 1, 30, 1e4], 400_000)).astype(np.float32)
    for s in (np.float32(0.0371), np.float32(1.7e-3)):
        q, _, _ = orc.quantize_groups(v, 1, 1, v.size, [0], 1, orc.SCALE_STATIC,
                                      np.array([s], np.float32))
        np.testing.assert_array_equal(q.astype(np.int64), _np_quant(v, s))


def test_quantizer_rounds_fp32_quotient_first(orc):
    """Where the exact quotient lies just below k + 1/2 but its binary32
    rounding equals k + 1/2, the definition (fp32 quotient first) gives the
    even neighbour; rounding the exact quotient would not.  Pairs are found by
    exact rational search."""
    rng = np.random.default_rng(3)
    found = 0
    for _ in range(20000):
        s = np.float32(rng.uniform(0.5, 2.0))
        k = int(rng.integers(1, 60))
        target = np.float32((k + 0.5) * float(s))
        for dv in (-2, -1, 1, 2):
            v = np.nextafter(target, np.float32(np.inf if dv > 0 else -np.inf), dtype=np.float32)
            if abs(dv) == 2:
                v = np.nextafter(v, np.float32(np.inf if dv > 0 else -np.inf), dtype=np.float32)
            exact = Fraction(float(v)) / Fraction(float(s))
            fq = np.float32(v) / np.float32(s)
            if fq == np.float32(k + 0.5) and exact != Fraction(2 * k + 1, 2):
                want = k if k % 2 == 0 else k + 1  # ties to even on the fp32 quotient
                q, _, _ = orc.quantize_groups(np.array([v], np.float32), 1, 1, 1, [0], 1,
                                              orc.SCALE_STATIC, np.array([s], np.float32))
                assert int(q[0]) == want
                naive = round(exact)  # Python rounds the exact rational
                if naive != want:
                    found += 1
        if found >= 5:
            break
    assert found >= 1


def test_quantizer_absmax_scales_and_groups(orc):
    rng = np.random.default_rng(11)
    outer, mid, inner, ng = 3, 10, 7, 4
    gmap = np.array([0, 1, 2, 3, 0, 1, 2, 3, 3, 3], np.int32)
    x = (rng.standard_normal((outer, mid, inner)) * 3).astype(np.float16)
    q, sc, nf = orc.quantize_groups(x, outer, mid, inner, gmap, ng, orc.SCALE_ABSMAX)
    assert nf == 0
    xf = x.astype(np.float32)
    for g in range(ng):
        am = np.abs(xf[:, gmap == g, :]).max()
        assert sc[g] == np.float32(am) / np.float32(127.0)  # numpy binary32 division
        np.testing.assert_array_equal(q[:, gmap == g, :].astype(np.int64),
                                      _np_quant(xf[:, gmap == g, :], sc[g]))
        # the largest magnitude of each group reaches +-127
        assert np.abs(q[:, gmap == g, :]).max() == 127


def test_quantizer_nonfinite_and_zero_group(orc):
    x = np.array([np.nan, np.inf, -np.inf, 1.0, 0.0, 0.0], np.float32)
    q, sc, nf = orc.quantize_groups(x, 1, 6, 1, [0, 0, 0, 0, 1, 1], 2, orc.SCALE_ABSMAX)
    assert nf == 3
    assert list(q) == [0, 0, 0, 127, 0, 0]
    assert sc[1] == 0.0


def test_quantizer_rejects_bad_group(orc):
    with pytest.raises(ValueError):
        orc.quantize_groups(np.zeros(4, np.float32), 1, 4, 1, [0, 1, 2, 5], 3, orc.SCALE_ABSMAX)


# ---- soft-edge codec ---------------------------------------------------------

def test_softedge_golden(orc):
    rows = [r.split() for r in golden_rows("softedge_cases.txt")]
    vals = np.array([float(r[0]) for r in rows], np.float32)
    codes, nf = orc.softedge_encode(vals, 1.0, 1.0, 63.0, 2)
    assert nf == 0
    for r, c in zip(rows, codes):
        assert int(c) == int(r[1], 16), r
    dec = orc.softedge_decode(np.array([int(r[1], 16) for r in rows], np.uint8), 1.0, 2)
    for r, d in zip(rows, dec):
        assert d == np.float32(float(r[2])), r


@pytest.mark.parametrize("s,lo,hi,r", [(0.05, 0.1, 3.0, 2), (1.0 / 63, 0.02, 1.0, 2),
                                       (0.2, 0.0, 12.0, 2), (0.05, 0.1, 3.0, 1)])
def test_softedge_invariants_all_f16(orc, s, lo, hi, r):
    s, lo, hi = np.float32(s), np.float32(lo), np.float32(hi)
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    v = bits.view(np.float16)
    v = v[np.isfinite(v)]
    codes, nf = orc.softedge_encode(v, s, lo, hi, r)
    assert nf == 0
    dec = orc.softedge_decode(codes, s, r).astype(np.float64)
    a = np.abs(v.astype(np.float64))
    # mode prefix: 0xxxxxxx <=> lo <= |v| <= hi ; 10 <=> |v| < lo ; 11 <=> |v| > hi
    std = (codes >> 7) == 0
    small = (codes >> 6) == 2
    large = (codes >> 6) == 3
    np.testing.assert_array_equal(std, (a >= lo) & (a <= hi))
    np.testing.assert_array_equal(small, a < lo)
    np.testing.assert_array_equal(large, a > hi)
    # error bounds: half a step of the chosen mode unless the payload
    # saturated, plus the one binary32 rounding of the quotient v / step that
    # the definition takes before rounding to an integer
    step = np.where(small, float(s) * 2.0 ** -r, np.where(large, float(s) * 2.0 ** r, float(s)))
    lim = np.where(std, 63, 31)
    unsat = a <= (lim + 0.5) * step * (1 - 1e-7)
    err = np.abs(dec - v.astype(np.float64))
    assert np.all(err[unsat] <= 0.5 * step[unsat] + a[unsat] * 2.0 ** -22 + 1e-30)
    # saturated values decode to the end of the mode's range, with v's sign
    sat = ~unsat
    np.testing.assert_allclose(np.abs(dec[sat]), (lim * step)[sat], rtol=1e-6)
    assert np.all(np.sign(dec[sat]) == np.sign(v[sat].astype(np.float64)))


def test_softedge_decode_all_codes_roundtrip(orc):
    """Every byte decodes to payload * step of its mode; re-encoding a decoded
    value whose magnitude lies inside its mode's range returns the byte."""
    s, lo, hi, r = np.float32(1.0), np.float32(0.3), np.float32(40.0), 2
    codes = np.arange(256, dtype=np.uint16).astype(np.uint8)
    dec = orc.softedge_decode(codes, s, r)
    for c, d in zip(codes, dec):
        c = int(c)
        if c < 0x80:
            q = c - 128 if c >= 64 else c
            assert d == np.float32(q)
        else:
            q = (c & 0x3F) - 64 if (c & 0x3F) >= 32 else (c & 0x3F)
            assert d == np.float32(q * (4.0 if c & 0x40 else 0.25))
    back, _ = orc.softedge_encode(dec, s, lo, hi, r)
    a = np.abs(dec)
    consistent = np.where(codes < 0x80, (a >= lo) & (a <= hi),
                          np.where(codes & 0x40, a > hi, a < lo))
    # payloads -64 (0x40) and -32 (0xA0, 0xE0) lie outside the symmetric
    # clamp range, so the encoder never emits them
    consistent &= ~np.isin(codes, [0x40, 0xA0, 0xE0])
    np.testing.assert_array_equal(back[consistent], codes[consistent])
    assert consistent.sum() > 100


def test_softedge_rejects_inverted_thresholds(orc):
    with pytest.raises(ValueError):
        orc.softedge_encode(np.zeros(4, np.float32), 1.0, 5.0, 1.0, 2)


def test_softedge_nonfinite(orc):
    codes, nf = orc.softedge_encode(np.array([np.nan, np.inf, 2.0], np.float32), 1.0, 0.5, 3.0, 2)
    assert nf == 2 and list(codes[:2]) == [0, 0] and codes[2] == 2


def test_half_conversion(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    for b in np.random.default_rng(0).choice(65536, 3000, replace=False):
        got = orc.half_to_double(int(b))
        if np.isnan(ref[b]):
            assert np.isnan(got)
        else:
            assert got == ref[b]
