"""ctypes front end of the CPU oracle -- TEST INFRASTRUCTURE, NOT THE PRODUCT.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg may
import this module.  It loads oracle/liboracle.so (plain C, double precision)
and converts numpy arrays to and from it.  Nothing here imports the product
package or the CUDA library.

Array conventions (the problem statement, shared with the GPU path only
through the seeded inputs):
  * binary16 tensors are numpy float16 arrays; the oracle reads their bits;
  * int8 codes are numpy int8, soft-edge codes numpy uint8;
  * scales, A, D, dt_bias, h0 are float32;
  * outputs y and h_final are float64.
"""
import ctypes as C
import os

import numpy as np

from . import build_oracle

_lib = None

_i64 = C.c_int64
_i32 = C.c_int32
_vp = C.c_void_p


class _M1(C.Structure):
    _fields_ = [("batch", _i64), ("seqlen", _i64), ("dim", _i64), ("dstate", _i64),
                ("ngroups", _i64), ("state_group_size", _i32), ("x_format", _i32),
                ("x", _vp), ("x_group", _vp), ("x_scale", _vp), ("se_scale", C.c_float),
                ("se_log2_ratio", _i32), ("dt", _vp), ("dt_bias", _vp), ("dt_softplus", _i32),
                ("A", _vp), ("D", _vp), ("z", _vp), ("B", _vp), ("C", _vp),
                ("B_scale", _vp), ("C_scale", _vp), ("h0", _vp)]


class _SSD(C.Structure):
    _fields_ = [("batch", _i64), ("seqlen", _i64), ("nheads", _i64), ("headdim", _i64),
                ("dstate", _i64), ("ngroups", _i64), ("state_group_size", _i32),
                ("x_format", _i32), ("x", _vp), ("x_group", _vp), ("x_scale", _vp),
                ("se_scale", C.c_float), ("se_log2_ratio", _i32), ("dt", _vp),
                ("dt_bias", _vp), ("dt_softplus", _i32), ("A", _vp), ("D", _vp), ("z", _vp),
                ("B", _vp), ("C", _vp), ("B_scale", _vp), ("C_scale", _vp), ("h0", _vp)]


class _DEC(C.Structure):
    _fields_ = [("batch", _i64), ("nheads", _i64), ("headdim", _i64), ("dstate", _i64),
                ("ngroups", _i64), ("state_group_size", _i32), ("x_format", _i32),
                ("x", _vp), ("x_group", _vp), ("x_scale", _vp), ("se_scale", C.c_float),
                ("se_log2_ratio", _i32), ("dt", _vp), ("dt_bias", _vp), ("dt_softplus", _i32),
                ("A", _vp), ("D", _vp), ("z", _vp), ("B", _vp), ("C", _vp),
                ("B_scale", _vp), ("C_scale", _vp)]


X_INT8_GROUP = 0
X_SOFTEDGE = 1
SCALE_STATIC = 0
SCALE_ABSMAX = 1


def lib():
    global _lib
    if _lib is None:
        # SSMQ_ORACLE_LIB points at an alternative build (the mutation tests
        # load deliberately broken copies through it)
        path = os.environ.get("SSMQ_ORACLE_LIB") or build_oracle.build()
        L = C.CDLL(path)
        L.orc_half_to_double.restype = C.c_double
        L.orc_half_to_double.argtypes = [C.c_uint16]
        L.orc_quantize_groups.restype = _i64
        L.orc_quantize_groups.argtypes = [_vp, _i32, _i64, _i64, _i64, _vp, _i32, _i32, _vp, _vp]
        L.orc_softedge_encode.restype = _i64
        L.orc_softedge_encode.argtypes = [_vp, _i32, _i64, C.c_float, C.c_float, C.c_float,
                                          _i32, _vp]
        L.orc_softedge_decode.restype = None
        L.orc_softedge_decode.argtypes = [_vp, _i64, C.c_float, _i32, _vp]
        L.orc_m1_scan.restype = _i32
        L.orc_m1_scan.argtypes = [C.POINTER(_M1), _i64, _vp, _vp, _vp, _i32]
        L.orc_m1_decode_step.restype = _i32
        L.orc_m1_decode_step.argtypes = [C.POINTER(_M1), _i64, _vp, _vp, _vp]
        L.orc_ssd_scan.restype = _i32
        L.orc_ssd_scan.argtypes = [C.POINTER(_SSD), _i64, _vp, _vp, _vp, _i32]
        L.orc_ssd_scan_chunked.restype = _i32
        L.orc_ssd_scan_chunked.argtypes = [C.POINTER(_SSD), _i64, _i64, _vp, _vp, _vp, _i32]
        L.orc_decode_step.restype = _i32
        L.orc_decode_step.argtypes = [C.POINTER(_DEC), _i64, _vp, _vp, _vp]
        L.orc_absmax_per_mid.restype = None
        L.orc_absmax_per_mid.argtypes = [_vp, _i32, _i64, _i64, _i64, _vp]
        L.orc_cluster_by_absmax.restype = _i32
        L.orc_cluster_by_absmax.argtypes = [_vp, _i64, _i32, _vp, _vp]
        L.orc_percentile_abs.restype = C.c_double
        L.orc_percentile_abs.argtypes = [_vp, _i32, _i64, C.c_double]
        L.orc_exp_f32_n.restype = None
        L.orc_exp_f32_n.argtypes = [_vp, _i64, _vp]
        L.orc_silu_f32_n.restype = None
        L.orc_silu_f32_n.argtypes = [_vp, _i64, _vp]
        L.orc_conv_silu.restype = _i64
        L.orc_conv_silu.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _vp, _vp]
        L.orc_softedge_thresholds.restype = None
        L.orc_softedge_thresholds.argtypes = [_vp, _i32, _i64, C.c_double, C.c_double,
                                              C.c_double, _vp]
        _lib = L
    return _lib


def default_threads():
    return max(1, os.cpu_count() or 1)


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=dtype)


def _src(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a, 1
    if a.dtype == np.float32:
        return a, 0
    raise TypeError("quantizer input must be float16 or float32")


# ---- quantizers -----------------------------------------------------------

def quantize_groups(src, outer, mid, inner, group_of_mid, n_groups, mode, scales=None):
    """Returns (q int8 same shape as src, scales float32[n_groups], n_nonfinite)."""
    s, is16 = _src(src)
    g = _c(group_of_mid, np.int32)
    if mode == SCALE_ABSMAX:
        sc = np.zeros(n_groups, np.float32)
    else:
        sc = _c(scales, np.float32).copy()
    q = np.zeros(s.shape, np.int8)
    r = lib().orc_quantize_groups(_p(s), is16, outer, mid, inner, _p(g), n_groups, mode,
                                  _p(sc), _p(q))
    if r < 0:
        raise ValueError("orc_quantize_groups: invalid arguments")
    return q, sc, int(r)


def softedge_encode(src, scale, thr_lo, thr_hi, log2_ratio=2):
    s, is16 = _src(src)
    codes = np.zeros(s.shape, np.uint8)
    r = lib().orc_softedge_encode(_p(s), is16, s.size, scale, thr_lo, thr_hi, log2_ratio,
                                  _p(codes))
    if r < 0:
        raise ValueError("orc_softedge_encode: invalid arguments")
    return codes, int(r)


def softedge_decode(codes, scale, log2_ratio=2):
    c = _c(codes, np.uint8)
    out = np.zeros(c.shape, np.float32)
    lib().orc_softedge_decode(_p(c), c.size, scale, log2_ratio, _p(out))
    return out


def half_to_double(bits):
    return lib().orc_half_to_double(int(bits))


# ---- scans ------------------------------------------------------------------

class _Keep:
    """Holds contiguous copies alive while the C call runs."""

    def __init__(self):
        self.items = []

    def __call__(self, a, dtype):
        a = _c(a, dtype)
        self.items.append(a)
        return _p(a)


def _units(units):
    if units is None:
        return None, 0
    u = np.ascontiguousarray(units, dtype=np.int64)
    return u, u.size


def _xfmt(x):
    return X_SOFTEDGE if x.dtype == np.uint8 else X_INT8_GROUP


def m1_scan(x, dt, A, B, C_, B_scale, C_scale, state_group_size, *, x_group=None,
            x_scale=None, se_scale=0.0, se_log2_ratio=2, D=None, z=None, dt_bias=None,
            dt_softplus=True, h0=None, ngroups=None, units=None, threads=None):
    """Mamba-1 selective scan.  x: (b, d, L) int8 or soft-edge uint8; B, C:
    (b, G, N, L).  Returns y [n_units, L] and h_final [n_units, N] (float64);
    units default to all (batch, channel) pairs."""
    k = _Keep()
    b, d, L = x.shape
    G, N = B.shape[1], B.shape[2]
    pr = _M1()
    pr.batch, pr.seqlen, pr.dim, pr.dstate, pr.ngroups = b, L, d, N, G
    pr.state_group_size = state_group_size
    pr.x_format = _xfmt(x)
    pr.x = k(x, x.dtype)
    pr.x_group = k(x_group, np.int32)
    pr.x_scale = k(x_scale, np.float32)
    pr.se_scale = se_scale
    pr.se_log2_ratio = se_log2_ratio
    pr.dt = k(dt, np.float16)
    pr.dt_bias = k(dt_bias, np.float32)
    pr.dt_softplus = int(bool(dt_softplus))
    pr.A = k(A, np.float32)
    pr.D = k(D, np.float32)
    pr.z = k(z, np.float16)
    pr.B = k(B, np.int8)
    pr.C = k(C_, np.int8)
    pr.B_scale = k(B_scale, np.float32)
    pr.C_scale = k(C_scale, np.float32)
    pr.h0 = k(h0, np.float32)
    u, nu = _units(units)
    if u is None:
        nu = b * d
    y = np.zeros((nu, L), np.float64)
    hf = np.zeros((nu, N), np.float64)
    r = lib().orc_m1_scan(C.byref(pr), nu, _p(u), _p(y), _p(hf),
                          threads or default_threads())
    if r != 0:
        raise ValueError("orc_m1_scan: invalid arguments")
    return y, hf


def m1_decode_step(state, x, dt, A, B, C_, B_scale, C_scale, state_group_size, *,
                   x_group=None, x_scale=None, se_scale=0.0, se_log2_ratio=2, D=None, z=None,
                   dt_bias=None, dt_softplus=True, units=None):
    """Mamba-1 single-token update.  state: float64 [n_units, N] (updated in
    place); x, dt, z: (b, d); B, C: (b, G, N).  Returns y [n_units]."""
    k = _Keep()
    b, d = x.shape
    G, N = B.shape[1], B.shape[2]
    pr = _M1()
    pr.batch, pr.seqlen, pr.dim, pr.dstate, pr.ngroups = b, 1, d, N, G
    pr.state_group_size = state_group_size
    pr.x_format = _xfmt(x)
    pr.x = k(x, x.dtype)
    pr.x_group = k(x_group, np.int32)
    pr.x_scale = k(x_scale, np.float32)
    pr.se_scale = se_scale
    pr.se_log2_ratio = se_log2_ratio
    pr.dt = k(dt, np.float16)
    pr.dt_bias = k(dt_bias, np.float32)
    pr.dt_softplus = int(bool(dt_softplus))
    pr.A = k(A, np.float32)
    pr.D = k(D, np.float32)
    pr.z = k(z, np.float16)
    pr.B = k(B, np.int8)
    pr.C = k(C_, np.int8)
    pr.B_scale = k(B_scale, np.float32)
    pr.C_scale = k(C_scale, np.float32)
    pr.h0 = None
    u, nu = _units(units)
    if u is None:
        nu = b * d
    assert state.dtype == np.float64 and state.flags.c_contiguous and state.size == nu * N
    y = np.zeros(nu, np.float64)
    r = lib().orc_m1_decode_step(C.byref(pr), nu, _p(u), _p(state), _p(y))
    if r != 0:
        raise ValueError("orc_m1_decode_step: invalid arguments")
    return y


def _ssd_problem(k, x, dt, A, B, C_, B_scale, C_scale, state_group_size, x_group, x_scale,
                 se_scale, se_log2_ratio, D, z, dt_bias, dt_softplus, h0):
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    pr = _SSD()
    pr.batch, pr.seqlen, pr.nheads, pr.headdim, pr.dstate, pr.ngroups = b, L, H, P, N, G
    pr.state_group_size = state_group_size
    pr.x_format = _xfmt(x)
    pr.x = k(x, x.dtype)
    pr.x_group = k(x_group, np.int32)
    pr.x_scale = k(x_scale, np.float32)
    pr.se_scale = se_scale
    pr.se_log2_ratio = se_log2_ratio
    pr.dt = k(dt, np.float16)
    pr.dt_bias = k(dt_bias, np.float32)
    pr.dt_softplus = int(bool(dt_softplus))
    pr.A = k(A, np.float32)
    pr.D = k(D, np.float32)
    pr.z = k(z, np.float16)
    pr.B = k(B, np.int8)
    pr.C = k(C_, np.int8)
    pr.B_scale = k(B_scale, np.float32)
    pr.C_scale = k(C_scale, np.float32)
    pr.h0 = k(h0, np.float32)
    return pr, (b, L, H, P, N)


def ssd_scan(x, dt, A, B, C_, B_scale, C_scale, state_group_size, *, x_group=None,
             x_scale=None, se_scale=0.0, se_log2_ratio=2, D=None, z=None, dt_bias=None,
             dt_softplus=True, h0=None, units=None, threads=None, chunk=None):
    """Mamba-2 SSD scan.  x: (b, L, H, P); dt: (b, L, H); B, C: (b, L, G, N).
    chunk=None runs the sequential definition; an integer runs the chunked
    form (self-check).  Returns y [n_units, L, P], h_final [n_units, P, N]."""
    k = _Keep()
    pr, (b, L, H, P, N) = _ssd_problem(k, x, dt, A, B, C_, B_scale, C_scale,
                                       state_group_size, x_group, x_scale, se_scale,
                                       se_log2_ratio, D, z, dt_bias, dt_softplus, h0)
    u, nu = _units(units)
    if u is None:
        nu = b * H
    y = np.zeros((nu, L, P), np.float64)
    hf = np.zeros((nu, P, N), np.float64)
    th = threads or default_threads()
    if chunk is None:
        r = lib().orc_ssd_scan(C.byref(pr), nu, _p(u), _p(y), _p(hf), th)
    else:
        r = lib().orc_ssd_scan_chunked(C.byref(pr), chunk, nu, _p(u), _p(y), _p(hf), th)
    if r != 0:
        raise ValueError("orc_ssd_scan: invalid arguments")
    return y, hf


def decode_step(state, x, dt, A, B, C_, B_scale, C_scale, state_group_size, *, x_group=None,
                x_scale=None, se_scale=0.0, se_log2_ratio=2, D=None, z=None, dt_bias=None,
                dt_softplus=True, units=None):
    """Mamba-2 single-token update.  state: float64 [n_units, P, N] (updated in
    place); x: (b, H, P); dt: (b, H); B, C: (b, G, N).  Returns y [n_units, P]."""
    k = _Keep()
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    pr = _DEC()
    pr.batch, pr.nheads, pr.headdim, pr.dstate, pr.ngroups = b, H, P, N, G
    pr.state_group_size = state_group_size
    pr.x_format = _xfmt(x)
    pr.x = k(x, x.dtype)
    pr.x_group = k(x_group, np.int32)
    pr.x_scale = k(x_scale, np.float32)
    pr.se_scale = se_scale
    pr.se_log2_ratio = se_log2_ratio
    pr.dt = k(dt, np.float16)
    pr.dt_bias = k(dt_bias, np.float32)
    pr.dt_softplus = int(bool(dt_softplus))
    pr.A = k(A, np.float32)
    pr.D = k(D, np.float32)
    pr.z = k(z, np.float16)
    pr.B = k(B, np.int8)
    pr.C = k(C_, np.int8)
    pr.B_scale = k(B_scale, np.float32)
    pr.C_scale = k(C_scale, np.float32)
    u, nu = _units(units)
    if u is None:
        nu = b * H
    assert state.dtype == np.float64 and state.flags.c_contiguous and state.size == nu * P * N
    y = np.zeros((nu, P), np.float64)
    r = lib().orc_decode_step(C.byref(pr), nu, _p(u), _p(state), _p(y))
    if r != 0:
        raise ValueError("orc_decode_step: invalid arguments")
    return y


# ---- calibration ------------------------------------------------------------

def absmax_per_mid(src, outer, mid, inner):
    s, is16 = _src(src)
    out = np.zeros(mid, np.float64)
    lib().orc_absmax_per_mid(_p(s), is16, outer, mid, inner, _p(out))
    return out


def cluster_by_absmax(absmax, k):
    a = _c(absmax, np.float64)
    cl = np.zeros(a.size, np.int32)
    sc = np.zeros(k, np.float32)
    if lib().orc_cluster_by_absmax(_p(a), a.size, k, _p(cl), _p(sc)) != 0:
        raise ValueError("orc_cluster_by_absmax: invalid arguments")
    return cl, sc


def percentile_abs(src, q):
    s, is16 = _src(src)
    return float(lib().orc_percentile_abs(_p(s), is16, s.size, q))


def softedge_thresholds(src, q_lo, q_hi, alpha, previous=(0.0, 0.0, 0.0)):
    """{scale, lo, hi} float32[3] after one threshold update."""
    s, is16 = _src(src)
    thr = np.asarray(previous, dtype=np.float32).copy()
    lib().orc_softedge_thresholds(_p(s), is16, s.size, q_lo, q_hi, alpha, _p(thr))
    return thr


# ---- causal depthwise convolution + SiLU (the producer of the scan input) --

def exp_f32(v):
    """The oracle's binary32 e^v (Cody-Waite reduction + Taylor polynomial)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty_like(v)
    lib().orc_exp_f32_n(_p(v), v.size, _p(out))
    return out


def silu_f32(a):
    """The oracle's binary32 silu(a) = a * fl32(1 / fl32(1 + e^-a))."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty_like(a)
    lib().orc_silu_f32_n(_p(a), a.size, _p(out))
    return out


def conv_silu(x, weight, bias=None, x_prev=None):
    """u = silu(causal depthwise conv(x)) in binary32 for x (b, d, L)
    float16, weight (d, W) float32, bias (d,) or None, x_prev (b, d, W-1)
    float16 or None.  Returns (u float32 (b, d, L), the next call's conv
    state float16 (b, d, W-1), number of non-finite u)."""
    x = np.ascontiguousarray(x, dtype=np.float16)
    b, d, L = x.shape
    w = np.ascontiguousarray(weight, dtype=np.float32)
    W = w.shape[1]
    bias = _c(bias, np.float32)
    x_prev = _c(x_prev, np.float16)
    u = np.empty((b, d, L), np.float32)
    st = np.empty((b, d, W - 1), np.float16)
    r = lib().orc_conv_silu(_p(x), _p(x_prev), _p(w), _p(bias), b, d, L, W, _p(u), _p(st))
    if r < 0:
        raise ValueError("orc_conv_silu: invalid arguments")
    return u, st, int(r)
