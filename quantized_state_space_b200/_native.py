"""ctypes binding of libssmq.so (include/ssmq.h): argument marshalling only.

Every function here has the name of the C entry point it calls.  Tensor
arguments may be torch tensors (their device pointer is passed), plain
integer addresses, or None (NULL).  A non-OK status raises SSMQError with the
library's message.  There is no fallback: if the shared library is missing
the import fails.
"""
import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libssmq.so")

OK, ERR_INVALID_ARG, ERR_ALIGNMENT, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_NONFINITE = range(7)
STATUS_NAMES = {0: "SSMQ_OK", 1: "SSMQ_ERR_INVALID_ARG", 2: "SSMQ_ERR_ALIGNMENT",
                3: "SSMQ_ERR_UNSUPPORTED", 4: "SSMQ_ERR_CUDA", 5: "SSMQ_ERR_TIMEOUT",
                6: "SSMQ_ERR_NONFINITE"}
DEV_NONFINITE, DEV_BAD_GROUP, DEV_BAD_SCALE, DEV_TIMEOUT = 1, 2, 4, 8
F32, F16 = 0, 1
SCALE_STATIC, SCALE_ABSMAX = 0, 1
X_INT8_GROUP, X_SOFTEDGE, X_F16_GROUP, X_F16_SOFTEDGE = 0, 1, 2, 3

_i64, _i32, _vp, _f32 = C.c_int64, C.c_int32, C.c_void_p, C.c_float


class SSMQError(RuntimeError):
    def __init__(self, status, message):
        super().__init__("%s: %s" % (STATUS_NAMES.get(status, status), message))
        self.status = status


class ScanArgs(C.Structure):
    _fields_ = [("batch", _i64), ("seqlen", _i64), ("dim", _i64), ("dstate", _i64),
                ("ngroups", _i64), ("state_group_size", _i32), ("x_format", _i32),
                ("x", _vp), ("x_group", _vp), ("x_scale", _vp), ("n_x_groups", _i32),
                ("se_scale", _f32), ("se_log2_ratio", _i32), ("dt", _vp), ("dt_bias", _vp),
                ("dt_softplus", _i32), ("A", _vp), ("D", _vp), ("z", _vp), ("B", _vp),
                ("C", _vp), ("B_scale", _vp), ("C_scale", _vp), ("h0", _vp), ("y", _vp),
                ("h_final", _vp), ("status", _vp), ("se_lo", _f32), ("se_hi", _f32),
                ("y_q", _vp), ("y_group", _vp), ("y_scale", _vp), ("n_y_groups", _i32),
                ("time_segments", _i32), ("workspace", _vp), ("workspace_bytes", C.c_size_t),
                ("dec_final", _vp)]


class SSDArgs(C.Structure):
    _fields_ = [("batch", _i64), ("seqlen", _i64), ("nheads", _i64), ("headdim", _i64),
                ("dstate", _i64), ("ngroups", _i64), ("chunk", _i64),
                ("state_group_size", _i32), ("x_format", _i32), ("x", _vp), ("x_group", _vp),
                ("x_scale", _vp), ("n_x_groups", _i32), ("se_scale", _f32),
                ("se_log2_ratio", _i32), ("dt", _vp), ("dt_bias", _vp), ("dt_softplus", _i32),
                ("A", _vp), ("D", _vp), ("z", _vp), ("B", _vp), ("C", _vp), ("B_scale", _vp),
                ("C_scale", _vp), ("h0", _vp), ("y", _vp), ("h_final", _vp), ("status", _vp), ("y_q", _vp),
                ("y_group", _vp), ("y_scale", _vp), ("n_y_groups", _i32),
                ("max_segments", _i32), ("dec_final", _vp)]


class DecodeArgs(C.Structure):
    _fields_ = [("batch", _i64), ("nheads", _i64), ("headdim", _i64), ("dstate", _i64),
                ("ngroups", _i64), ("state_group_size", _i32), ("x_format", _i32),
                ("x", _vp), ("x_group", _vp), ("x_scale", _vp), ("n_x_groups", _i32),
                ("se_scale", _f32), ("se_log2_ratio", _i32), ("dt", _vp), ("dt_bias", _vp),
                ("dt_softplus", _i32), ("A", _vp), ("D", _vp), ("z", _vp), ("B", _vp),
                ("C", _vp), ("B_scale", _vp), ("C_scale", _vp), ("state", _vp), ("y", _vp),
                ("status", _vp)]


class M1DecodeArgs(C.Structure):
    _fields_ = [("batch", _i64), ("dim", _i64), ("dstate", _i64), ("ngroups", _i64),
                ("state_group_size", _i32), ("x_format", _i32), ("x", _vp), ("x_group", _vp),
                ("x_scale", _vp), ("n_x_groups", _i32), ("se_scale", _f32),
                ("se_log2_ratio", _i32), ("dt", _vp), ("dt_bias", _vp), ("dt_softplus", _i32),
                ("A", _vp), ("D", _vp), ("z", _vp), ("B", _vp), ("C", _vp), ("B_scale", _vp),
                ("C_scale", _vp), ("state", _vp), ("y", _vp), ("status", _vp)]


class ConvArgs(C.Structure):
    _fields_ = [("batch", _i64), ("seqlen", _i64), ("dim", _i64), ("width", _i32), ("x", _vp),
                ("weight", _vp), ("bias", _vp), ("x_prev", _vp), ("out_format", _i32),
                ("x_group", _vp), ("x_scale", _vp), ("n_x_groups", _i32), ("se_scale", _f32),
                ("se_lo", _f32), ("se_hi", _f32), ("se_log2_ratio", _i32), ("codes", _vp),
                ("u", _vp), ("x_prev_out", _vp), ("status", _vp)]


# entry point -> (restype, argtypes); every name declared in include/ssmq.h
class QuantJob(C.Structure):
    _fields_ = [("src", _vp), ("dtype", _i32), ("outer", _i64), ("mid", _i64), ("inner", _i64),
                ("group_of_mid", _vp), ("n_groups", _i32), ("scales", _vp), ("q_out", _vp)]


SIGNATURES = {
    "ssmq_quantize_groups_batch": (_i32, [C.POINTER(QuantJob), _i32, _vp, _vp]),
    "ssmq_state_chain": (_i32, [_vp, _vp, _i32, _i64, _i64, _vp, _vp]),
    "ssmq_ssd_carry_in": (_i32, [C.c_void_p, _vp, _vp, C.c_size_t, _vp]),
    "ssmq_quantize_groups": (_i32, [_vp, _i32, _i64, _i64, _i64, _vp, _i32, _i32, _vp, _vp,
                                    _vp, _vp]),
    "ssmq_softedge_encode": (_i32, [_vp, _i32, _i64, _f32, _f32, _f32, _i32, _vp, _vp, _vp]),
    "ssmq_softedge_decode": (_i32, [_vp, _i64, _f32, _i32, _vp, _vp]),
    "ssmq_selective_scan_w8": (_i32, [C.POINTER(ScanArgs), _vp]),
    "ssmq_scan_time_segments": (_i32, [C.POINTER(ScanArgs)]),
    "ssmq_selective_scan_carry_in": (_i32, [C.POINTER(ScanArgs), _vp, _vp]),
    "ssmq_scan_workspace_size": (C.c_size_t, [C.POINTER(ScanArgs)]),
    "ssmq_conv_silu_quantize": (_i32, [C.POINTER(ConvArgs), _vp]),
    "ssmq_ssd_workspace_size": (C.c_size_t, [C.POINTER(SSDArgs)]),
    "ssmq_ssd_chunk_scan_w8": (_i32, [C.POINTER(SSDArgs), _vp, C.c_size_t, _vp]),
    "ssmq_state_update_w8": (_i32, [C.POINTER(DecodeArgs), _vp]),
    "ssmq_selective_state_update_w8": (_i32, [C.POINTER(M1DecodeArgs), _vp]),
    "ssmq_group_absmax": (_i32, [_vp, _i32, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _vp]),
    "ssmq_cluster_by_absmax": (_i32, [_vp, _i64, _i32, _vp, _vp, _vp, _vp]),
    "ssmq_percentile_workspace_size": (C.c_size_t, []),
    "ssmq_percentile_abs": (_i32, [_vp, _i32, _i64, C.POINTER(C.c_double), _i32, _vp, _vp,
                                   C.c_size_t, _vp]),
    "ssmq_softedge_calibrate": (_i32, [_vp, _i32, _i64, C.c_double, C.c_double, _f32, _vp, _vp,
                                       C.c_size_t, _vp]),
    "ssmq_percentile_abs_noalloc": (_i32, [_vp, _i32, _i64, C.POINTER(C.c_double), _i32, _vp,
                                           _vp]),
    "ssmq_softedge_calibrate_noalloc": (_i32, [_vp, _i32, _i64, C.c_double, C.c_double, _f32,
                                               _vp, _vp]),
    "ssmq_probe_ex2": (_i32, [_i32, _vp, C.POINTER(C.c_int64), _vp]),
    "ssmq_last_error": (C.c_char_p, []),
    "ssmq_version": (_i32, []),
}

_lib = None


def lib():
    """Loads libssmq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libssmq.so is not built; run `python -m "
                              "quantized_state_space_b200.build_native` (or "
                              "__graft_entry__.build())")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def ptr(t):
    """Device address of a tensor / int / None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    if torch.cuda.is_available() and torch.cuda.is_initialized():
        return torch.cuda.current_stream().cuda_stream
    return None


def _dtype_of(t, dtype):
    if dtype is not None:
        return dtype
    import torch
    if t.dtype == torch.float16:
        return F16
    if t.dtype == torch.float32:
        return F32
    raise TypeError("source must be float16 or float32")


def _check(status):
    if status != OK:
        raise SSMQError(status, lib().ssmq_last_error().decode())


def ssmq_last_error():
    return lib().ssmq_last_error().decode()


def ssmq_version():
    return lib().ssmq_version()


def ssmq_probe_ex2(iters, sink, stream=None):
    """Launches the exp2 throughput probe; returns the number of exponentials."""
    n = C.c_int64(0)
    _check(lib().ssmq_probe_ex2(int(iters), ptr(sink), C.byref(n), _stream(stream)))
    return int(n.value)


def ssmq_quantize_groups(src, outer, mid, inner, group_of_mid, n_groups, mode, scales, q_out,
                         status=None, stream=None, dtype=None):
    _check(lib().ssmq_quantize_groups(ptr(src), _dtype_of(src, dtype), outer, mid, inner,
                                      ptr(group_of_mid), n_groups, mode, ptr(scales), ptr(q_out),
                                      ptr(status), _stream(stream)))


def ssmq_quantize_groups_batch(jobs, status=None, stream=None):
    """jobs: list of dicts with the fields of ssmq_quant_job (tensors for the
    pointer fields; dtype taken from src when absent)."""
    arr = (QuantJob * len(jobs))(*[
        QuantJob(ptr(j["src"]), j.get("dtype", None) or _dtype_of(j["src"], None), j["outer"],
                 j["mid"], j["inner"], ptr(j["group_of_mid"]), j["n_groups"], ptr(j["scales"]),
                 ptr(j["q_out"])) for j in jobs])
    _check(lib().ssmq_quantize_groups_batch(arr, len(jobs), ptr(status), _stream(stream)))


def ssmq_softedge_encode(src, n, scale, thr_lo, thr_hi, log2_ratio, codes, status=None,
                         stream=None, dtype=None):
    _check(lib().ssmq_softedge_encode(ptr(src), _dtype_of(src, dtype), n, scale, thr_lo, thr_hi,
                                      log2_ratio, ptr(codes), ptr(status), _stream(stream)))


def ssmq_softedge_decode(codes, n, scale, log2_ratio, out, stream=None):
    _check(lib().ssmq_softedge_decode(ptr(codes), n, scale, log2_ratio, ptr(out),
                                      _stream(stream)))


_FIELD_TYPES = {}


def _fill(struct_cls, fields):
    types = _FIELD_TYPES.get(struct_cls)
    if types is None:
        types = _FIELD_TYPES[struct_cls] = dict(struct_cls._fields_)
    a = struct_cls()
    for k, v in fields.items():
        ftype = types.get(k)
        if ftype is None:
            raise TypeError("unknown field %r for %s" % (k, struct_cls.__name__))
        setattr(a, k, ptr(v) if ftype is _vp else v)
    return a


def ssmq_selective_scan_w8(stream=None, **fields):
    """Fields of ssmq_scan_args as keywords (tensors for pointer fields)."""
    a = _fill(ScanArgs, fields)
    _check(lib().ssmq_selective_scan_w8(C.byref(a), _stream(stream)))


def ssmq_selective_scan_carry_in(h_carry, stream=None, **fields):
    """Fields of ssmq_scan_args as keywords; h_carry the carried state."""
    a = _fill(ScanArgs, fields)
    _check(lib().ssmq_selective_scan_carry_in(C.byref(a), ptr(h_carry), _stream(stream)))


def ssmq_scan_time_segments(**fields):
    return int(lib().ssmq_scan_time_segments(C.byref(_fill(ScanArgs, fields))))


def ssmq_scan_workspace_size(**fields):
    return int(lib().ssmq_scan_workspace_size(C.byref(_fill(ScanArgs, fields))))


def ssmq_conv_silu_quantize(stream=None, **fields):
    """Fields of ssmq_conv_args as keywords (tensors for pointer fields)."""
    a = _fill(ConvArgs, fields)
    _check(lib().ssmq_conv_silu_quantize(C.byref(a), _stream(stream)))


def ssmq_ssd_workspace_size(**fields):
    return int(lib().ssmq_ssd_workspace_size(C.byref(_fill(SSDArgs, fields))))


def ssmq_ssd_chunk_scan_w8(workspace=None, ws_bytes=0, stream=None, **fields):
    a = _fill(SSDArgs, fields)
    _check(lib().ssmq_ssd_chunk_scan_w8(C.byref(a), ptr(workspace), ws_bytes, _stream(stream)))


def ssmq_ssd_carry_in(h_carry, workspace=None, ws_bytes=0, stream=None, **fields):
    a = _fill(SSDArgs, fields)
    _check(lib().ssmq_ssd_carry_in(C.addressof(a), ptr(h_carry), ptr(workspace), ws_bytes,
                                   _stream(stream)))


def ssmq_state_chain(h_end, dec, n_parts, units, elems, h_out, stream=None):
    _check(lib().ssmq_state_chain(ptr(h_end), ptr(dec), n_parts, units, elems, ptr(h_out),
                                  _stream(stream)))


def ssmq_state_update_w8(stream=None, **fields):
    a = _fill(DecodeArgs, fields)
    _check(lib().ssmq_state_update_w8(C.byref(a), _stream(stream)))


def ssmq_selective_state_update_w8(stream=None, **fields):
    a = _fill(M1DecodeArgs, fields)
    _check(lib().ssmq_selective_state_update_w8(C.byref(a), _stream(stream)))


def ssmq_group_absmax(src, outer, mid, inner, group_of_mid, n_groups, absmax, status=None,
                      stream=None, dtype=None):
    _check(lib().ssmq_group_absmax(ptr(src), _dtype_of(src, dtype), outer, mid, inner,
                                   ptr(group_of_mid), n_groups, ptr(absmax), ptr(status),
                                   _stream(stream)))


def ssmq_cluster_by_absmax(absmax, n, k, cluster_of, scales, status=None, stream=None):
    _check(lib().ssmq_cluster_by_absmax(ptr(absmax), n, k, ptr(cluster_of), ptr(scales),
                                        ptr(status), _stream(stream)))


def ssmq_percentile_workspace_size():
    return int(lib().ssmq_percentile_workspace_size())


def ssmq_percentile_abs(src, n, q, out, workspace, ws_bytes, stream=None, dtype=None):
    qa = (C.c_double * len(q))(*[float(v) for v in q])
    _check(lib().ssmq_percentile_abs(ptr(src), _dtype_of(src, dtype), n, qa, len(q), ptr(out),
                                     ptr(workspace), ws_bytes, _stream(stream)))


def ssmq_softedge_calibrate(src, n, q_lo, q_hi, alpha, thresholds, workspace, ws_bytes,
                            stream=None, dtype=None):
    _check(lib().ssmq_softedge_calibrate(ptr(src), _dtype_of(src, dtype), n, float(q_lo),
                                         float(q_hi), float(alpha), ptr(thresholds),
                                         ptr(workspace), ws_bytes, _stream(stream)))


def ssmq_percentile_abs_noalloc(src, n, q, out, stream=None, dtype=None):
    qa = (C.c_double * len(q))(*[float(v) for v in q])
    _check(lib().ssmq_percentile_abs_noalloc(ptr(src), _dtype_of(src, dtype), n, qa, len(q),
                                             ptr(out), _stream(stream)))


def ssmq_softedge_calibrate_noalloc(src, n, q_lo, q_hi, alpha, thresholds, stream=None,
                                    dtype=None):
    _check(lib().ssmq_softedge_calibrate_noalloc(ptr(src), _dtype_of(src, dtype), n, float(q_lo),
                                                 float(q_hi), float(alpha), ptr(thresholds),
                                                 _stream(stream)))
