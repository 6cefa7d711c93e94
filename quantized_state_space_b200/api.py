"""User-facing calls on torch CUDA tensors.

Each function allocates its outputs with torch (device memory and streams are
PyTorch's job) and calls one C-ABI entry point through ``_native``; every step
of the computation runs in the CUDA library.  Layouts and semantics are those
of include/ssmq.h.
"""
import contextlib

import torch

from . import _native as N


def _dev_check(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _out(t, name, dtype, numel, device):
    """A caller-supplied tensor that the call writes (or reads whole): it must
    be contiguous, on the inputs' device, of the dtype and element count the
    kernels use, since the library cannot see the size behind a pointer."""
    if t is None:
        return
    if t.device != device or not t.is_contiguous():
        raise ValueError("%s must be a contiguous tensor on %s" % (name, device))
    if t.dtype != dtype or t.numel() != numel:
        raise ValueError("%s must be %s with %d elements (got %s with %d)"
                         % (name, dtype, numel, t.dtype, t.numel()))


def _in(t, name, dtypes, numel, device):
    """A caller-supplied tensor that the call reads: on the call's device,
    contiguous, of one of ``dtypes`` and with the element count the kernels
    read (the library reads that many elements behind the pointer)."""
    if t is None:
        return
    if not isinstance(dtypes, tuple):
        dtypes = (dtypes,)
    if t.device != device or not t.is_contiguous():
        raise ValueError("%s must be a contiguous tensor on %s" % (name, device))
    if t.dtype not in dtypes or (numel is not None and t.numel() != numel):
        raise ValueError("%s must be %s with %s elements (got %s with %d)"
                         % (name, "/".join(str(d) for d in dtypes),
                            "any number of" if numel is None else numel, t.dtype, t.numel()))


def _on(device):
    """Launches go to the device that holds the tensors (and its current
    stream), whatever device is current in the caller."""
    if device.type == "cuda":
        return torch.cuda.device(device)
    return contextlib.nullcontext()


_FP = (torch.float16, torch.float32)


def _status(t, device):
    """The optional device status word: 32-bit, at least one element."""
    if t is None:
        return
    if t.device != device or t.element_size() != 4 or t.numel() < 1:
        raise ValueError("status must be a 32-bit tensor of at least one element on %s" % device)


def _workspace(t, nbytes, device):
    """A caller-supplied workspace: uint8 bytes on the device, room for the
    256-byte alignment of its start."""
    if t is None or not nbytes:
        return
    if t.device != device or t.dtype != torch.uint8 or t.numel() < nbytes + 255:
        raise ValueError("workspace must be a uint8 tensor of at least %d bytes on %s"
                         % (nbytes + 255, device))


def _x_in(x, x_group, x_scale, channels, device, codes_only=False, se_lo=None):
    """x and its cluster map: int8 codes, soft-edge uint8 codes, or (Mamba-1
    scan only) binary16 activations, soft-edge encoded when thresholds are
    given; int8 codes and group-quantized binary16 x need the cluster map (one
    int32 entry per channel) and a scale table of at least one fp32 entry."""
    _in(x, "x", (torch.int8, torch.uint8) if codes_only else
        (torch.int8, torch.uint8, torch.float16), None, device)
    if x.dtype == torch.int8 or (x.dtype == torch.float16 and se_lo is None):
        _in(x_group, "x_group", torch.int32, channels, device)
        _in(x_scale, "x_scale", torch.float32, None, device)
        if x_group is None or x_scale is None or x_scale.numel() < 1:
            raise ValueError("x_group and a non-empty x_scale are required for int8 / binary16 x")


def _bc_in(B, C, B_scale, C_scale, numel, n_scales, device):
    _in(B, "B", torch.int8, numel, device)
    _in(C, "C", torch.int8, numel, device)
    _in(B_scale, "B_scale", torch.float32, n_scales, device)
    _in(C_scale, "C_scale", torch.float32, n_scales, device)


def _n_scales(G, Nst, state_group_size):
    if state_group_size < 1 or Nst % state_group_size:
        raise ValueError("dstate must be a multiple of state_group_size >= 1")
    return G * Nst // state_group_size


def quantize_groups(src, outer, mid, inner, group_of_mid, n_groups, *, scales=None,
                    absmax=False, out=None, status=None):
    """int8 codes of ``src`` (float16/float32) with one scale per group.
    absmax=True computes the scales (returned); else ``scales`` are used."""
    _dev_check(src, group_of_mid, scales)
    dv = src.device
    _in(src, "src", _FP, outer * mid * inner, dv)
    _in(group_of_mid, "group_of_mid", torch.int32, mid, dv)
    if not absmax:
        _in(scales, "scales", torch.float32, n_groups, dv)
    _out(out, "out", torch.int8, outer * mid * inner, dv)
    _status(status, dv)
    with _on(dv):
        q = out if out is not None else torch.empty(src.shape, dtype=torch.int8, device=dv)
        if absmax:
            scales = torch.empty(n_groups, dtype=torch.float32, device=dv)
        N.ssmq_quantize_groups(src, outer, mid, inner, group_of_mid, n_groups,
                               N.SCALE_ABSMAX if absmax else N.SCALE_STATIC, scales, q,
                               status=status)
    return q, scales


def quantize_groups_batch(jobs, *, status=None):
    """Static int8 codes of several tensors in one launch (per dtype and
    layout class).  jobs: sequence of (src, outer, mid, inner, group_of_mid,
    n_groups, scales, out-or-None); returns the code tensors."""
    outs, descs = [], []
    jobs = list(jobs)
    if not jobs:
        raise ValueError("at least one job")
    dv = jobs[0][0].device
    for src, outer, mid, inner, gmap, n_groups, scales, out in jobs:
        _dev_check(src, gmap, scales)
        _in(src, "src", _FP, outer * mid * inner, dv)
        _in(gmap, "group_of_mid", torch.int32, mid, dv)
        _in(scales, "scales", torch.float32, n_groups, dv)
        _out(out, "out", torch.int8, outer * mid * inner, dv)
        _status(status, dv)
        q = out if out is not None else torch.empty(src.shape, dtype=torch.int8, device=dv)
        outs.append(q)
        descs.append(dict(src=src, outer=outer, mid=mid, inner=inner, group_of_mid=gmap,
                          n_groups=n_groups, scales=scales, q_out=q))
    with _on(dv):
        N.ssmq_quantize_groups_batch(descs, status=status)
    return outs


def softedge_encode(src, scale, thr_lo, thr_hi, log2_ratio=2, *, out=None, status=None):
    _dev_check(src)
    _in(src, "src", _FP, None, src.device)
    _out(out, "out", torch.uint8, src.numel(), src.device)
    _status(status, src.device)
    with _on(src.device):
        codes = out if out is not None else torch.empty(src.shape, dtype=torch.uint8,
                                                        device=src.device)
        N.ssmq_softedge_encode(src, src.numel(), float(scale), float(thr_lo), float(thr_hi),
                               log2_ratio, codes, status=status)
    return codes


def softedge_decode(codes, scale, log2_ratio=2, *, out=None):
    _dev_check(codes)
    _in(codes, "codes", torch.uint8, None, codes.device)
    _out(out, "out", torch.float32, codes.numel(), codes.device)
    with _on(codes.device):
        o = out if out is not None else torch.empty(codes.shape, dtype=torch.float32,
                                                    device=codes.device)
        N.ssmq_softedge_decode(codes, codes.numel(), float(scale), log2_ratio, o)
    return o


def _x_fields(x, x_group, x_scale, se_scale, se_log2_ratio, se_lo=None, se_hi=None):
    """x format from the tensor: uint8 soft-edge codes, int8 codes, or
    binary16 activations encoded inside the kernel (soft-edge when thresholds
    are given, else the static group quantizer)."""
    if x.dtype == torch.uint8:
        return dict(x_format=N.X_SOFTEDGE, x=x, se_scale=float(se_scale),
                    se_log2_ratio=se_log2_ratio, n_x_groups=0)
    if x.dtype == torch.float16 and se_lo is not None:
        return dict(x_format=N.X_F16_SOFTEDGE, x=x, se_scale=float(se_scale),
                    se_log2_ratio=se_log2_ratio, n_x_groups=0, se_lo=float(se_lo),
                    se_hi=float(se_hi))
    fmt = N.X_F16_GROUP if x.dtype == torch.float16 else N.X_INT8_GROUP
    return dict(x_format=fmt, x=x, x_group=x_group, x_scale=x_scale,
                n_x_groups=int(x_scale.numel()), se_log2_ratio=se_log2_ratio)


def _y_fields(shape, device, y_group, y_scale, y_q, want_y, y, channels):
    """Optional int8 output (static per-cluster scales) and the binary16 y."""
    f = {}
    n = 1
    for v in shape:
        n *= v
    _out(y, "y", torch.float16, n, device)
    _out(y_q, "y_q", torch.int8, n, device)
    if y_group is not None:
        _dev_check(y_group, y_scale)
        _in(y_group, "y_group", torch.int32, channels, device)
        _in(y_scale, "y_scale", torch.float32, None, device)
        if y_scale is None or y_scale.numel() < 1:
            raise ValueError("y_group needs a non-empty y_scale")
        if y_q is None:
            y_q = torch.empty(shape, dtype=torch.int8, device=device)
        f = dict(y_q=y_q, y_group=y_group, y_scale=y_scale, n_y_groups=int(y_scale.numel()))
    if want_y and y is None:
        y = torch.empty(shape, dtype=torch.float16, device=device)
    return (y if want_y else None), y_q, f


def selective_scan(x, dt, A, B, C, B_scale, C_scale, state_group_size, *, x_group=None,
                   x_scale=None, se_scale=0.0, se_log2_ratio=2, se_lo=None, se_hi=None, D=None,
                   z=None, dt_bias=None, dt_softplus=True, h0=None, y=None, h_final=None,
                   return_state=True, y_group=None, y_scale=None, y_q=None, want_y=True,
                   time_segments=1, workspace=None, dec_final=None, status=None):
    """Mamba-1 W8A8 selective scan.  x (b, d, L) int8 codes, soft-edge uint8
    codes, or float16 activations that the kernel encodes itself (with
    x_group / x_scale, or with se_scale / se_lo / se_hi); dt, z (b, d, L)
    float16; B, C (b, G, N, L) int8.  Returns (y, h_final), or (y, h_final,
    y_q) when y_group / y_scale ask for the int8 output (y is None when
    want_y is False).  time_segments > 1 cuts L into that many segments
    scanned in parallel plus a carry-in pass (include/ssmq.h); the workspace
    it needs (uint8 bytes on the device) is allocated when not given.
    dec_final (b, d, N) float32, when given, receives the call's log2 decays
    A log2(e) sum_t delta_t (for chaining slices of a sequence)."""
    b, d, L = x.shape
    G, Nst = B.shape[1], B.shape[2]
    _dev_check(x, dt, A, B, C, B_scale, C_scale, x_group, x_scale, D, z, dt_bias, h0)
    dv = x.device
    _x_in(x, x_group, x_scale, d, dv, se_lo=se_lo)
    _in(dt, "dt", torch.float16, b * d * L, dv)
    _in(z, "z", torch.float16, b * d * L, dv)
    _in(A, "A", torch.float32, d * Nst, dv)
    _in(D, "D", torch.float32, d, dv)
    _in(dt_bias, "dt_bias", torch.float32, d, dv)
    _bc_in(B, C, B_scale, C_scale, b * G * Nst * L, _n_scales(G, Nst, state_group_size), dv)
    _in(h0, "h0", torch.float32, b * d * Nst, dv)
    _out(h_final, "h_final", torch.float32, b * d * Nst, dv)
    _out(dec_final, "dec_final", torch.float32, b * d * Nst, dv)
    _status(status, dv)
    with _on(dv):
        y, y_q, yf = _y_fields((b, d, L), dv, y_group, y_scale, y_q, want_y, y, d)
        if h_final is None and return_state:
            h_final = torch.empty((b, d, Nst), dtype=torch.float32, device=dv)
        fields = dict(batch=b, seqlen=L, dim=d, dstate=Nst, ngroups=G,
                      state_group_size=state_group_size,
                      **_x_fields(x, x_group, x_scale, se_scale, se_log2_ratio, se_lo, se_hi),
                      dt=dt, dt_bias=dt_bias, dt_softplus=int(bool(dt_softplus)), A=A, D=D, z=z,
                      B=B, C=C, B_scale=B_scale, C_scale=C_scale, h0=h0, y=y, h_final=h_final,
                      status=status, time_segments=int(time_segments), dec_final=dec_final,
                      **yf)
        # (one pass needs no workspace: no size query on that path)
        ws = N.ssmq_scan_workspace_size(**fields) if int(time_segments) > 1 else 0
        _workspace(workspace, ws, dv)
        if ws and workspace is None:
            workspace = torch.empty(ws + 256, dtype=torch.uint8, device=dv)
        wptr = (workspace.data_ptr() + 255) // 256 * 256 if ws else None
        N.ssmq_selective_scan_w8(workspace=wptr, workspace_bytes=ws, **fields)
    return (y, h_final, y_q) if yf else (y, h_final)


def selective_scan_carry_in(x, dt, A, B, C, B_scale, C_scale, state_group_size, h_carry, y, *,
                            D=None, z=None, dt_bias=None, dt_softplus=True, h_final=None,
                            status=None):
    """Adds the contribution of the start state h_carry (b, d, N) to the y
    (in place) and h_final (in place, if given) of a Mamba-1 scan call on the
    same inputs that started from a zero state.  x gives the shapes only."""
    _dev_check(x, dt, A, B, C, B_scale, C_scale, D, z, dt_bias, h_carry, y, h_final)
    b, d, L = x.shape
    G, Nst = B.shape[1], B.shape[2]
    dv = x.device
    _in(dt, "dt", torch.float16, b * d * L, dv)
    _in(z, "z", torch.float16, b * d * L, dv)
    _in(A, "A", torch.float32, d * Nst, dv)
    _in(D, "D", torch.float32, d, dv)
    _in(dt_bias, "dt_bias", torch.float32, d, dv)
    _bc_in(B, C, B_scale, C_scale, b * G * Nst * L, _n_scales(G, Nst, state_group_size), dv)
    _out(y, "y", torch.float16, b * d * L, dv)
    _out(h_carry, "h_carry", torch.float32, b * d * Nst, dv)
    _out(h_final, "h_final", torch.float32, b * d * Nst, dv)
    _status(status, dv)
    with _on(dv):
        N.ssmq_selective_scan_carry_in(h_carry, batch=b, seqlen=L, dim=d, dstate=Nst, ngroups=G,
                                       state_group_size=state_group_size, dt=dt,
                                       dt_bias=dt_bias, dt_softplus=int(bool(dt_softplus)), A=A,
                                       D=D, z=z, B=B, C=C, B_scale=B_scale, C_scale=C_scale, y=y,
                                       h_final=h_final, status=status)
    return y, h_final


def conv_silu_quantize(x, weight, *, bias=None, x_prev=None, x_group=None, x_scale=None,
                       se_scale=None, se_lo=None, se_hi=None, se_log2_ratio=2, codes=None,
                       want_u=False, u=None, x_prev_out=None, want_state=False, status=None):
    """The scan input's codes straight from the convolution's input: causal
    depthwise conv (weight (d, W), W <= 4; bias (d,); conv state x_prev
    (b, d, W-1)) + SiLU + the group quantizer (x_group / x_scale: int8
    codes) or the soft-edge encoder (se_scale / se_lo / se_hi: uint8 codes).
    x (b, d, L) float16.  Returns codes, plus u (float32 values coded) when
    want_u, plus the next call's state (b, d, W-1) float16 when want_state."""
    _dev_check(x, weight, bias, x_prev, x_group, x_scale)
    b, d, L = x.shape
    dv = x.device
    W = weight.shape[-1] if weight.dim() == 2 else 0
    _in(x, "x", torch.float16, b * d * L, dv)
    _in(weight, "weight", torch.float32, d * W, dv)
    _in(bias, "bias", torch.float32, d, dv)
    _in(x_prev, "x_prev", torch.float16, b * d * max(W - 1, 0), dv)
    soft = se_scale is not None
    if soft:
        cdt = torch.uint8
        fmt = dict(out_format=N.X_SOFTEDGE, se_scale=float(se_scale), se_lo=float(se_lo),
                   se_hi=float(se_hi), se_log2_ratio=se_log2_ratio)
    else:
        _in(x_group, "x_group", torch.int32, d, dv)
        _in(x_scale, "x_scale", torch.float32, None, dv)
        if x_group is None or x_scale is None or x_scale.numel() < 1:
            raise ValueError("x_group and a non-empty x_scale, or the soft-edge parameters, "
                             "are required")
        cdt = torch.int8
        fmt = dict(out_format=N.X_INT8_GROUP, x_group=x_group, x_scale=x_scale,
                   n_x_groups=int(x_scale.numel()))
    _out(codes, "codes", cdt, b * d * L, dv)
    _out(u, "u", torch.float32, b * d * L, dv)
    _out(x_prev_out, "x_prev_out", torch.float16, b * d * max(W - 1, 0), dv)
    _status(status, dv)
    with _on(dv):
        if codes is None:
            codes = torch.empty((b, d, L), dtype=cdt, device=dv)
        if want_u and u is None:
            u = torch.empty((b, d, L), dtype=torch.float32, device=dv)
        if want_state and x_prev_out is None:
            x_prev_out = torch.empty((b, d, max(W - 1, 0)), dtype=torch.float16, device=dv)
        N.ssmq_conv_silu_quantize(batch=b, seqlen=L, dim=d, width=W, x=x, weight=weight,
                                  bias=bias, x_prev=x_prev, codes=codes,
                                  u=u if want_u or u is not None else None,
                                  x_prev_out=x_prev_out, status=status, **fmt)
    out = (codes,)
    if want_u:
        out += (u,)
    if want_state:
        out += (x_prev_out,)
    return out if len(out) > 1 else codes


def _ssd_inputs(x, dt, A, B, C, B_scale, C_scale, state_group_size, x_group, x_scale, D, z,
                dt_bias, h0):
    b, L, H, P = x.shape
    G, Nst = B.shape[2], B.shape[3]
    dv = x.device
    _x_in(x, x_group, x_scale, H * P, dv, codes_only=True)
    _in(dt, "dt", torch.float16, b * L * H, dv)
    _in(z, "z", torch.float16, b * L * H * P, dv)
    for t, name in ((A, "A"), (D, "D"), (dt_bias, "dt_bias")):
        _in(t, name, torch.float32, H, dv)
    _bc_in(B, C, B_scale, C_scale, b * L * G * Nst, _n_scales(G, Nst, state_group_size), dv)
    _in(h0, "h0", torch.float32, b * H * P * Nst, dv)


def _ssd_call(x, dt, A, B, C, B_scale, C_scale, state_group_size, chunk, x_group, x_scale,
              se_scale, se_log2_ratio, D, z, dt_bias, dt_softplus, h0, y, h_final,
              max_segments, workspace, status, dec_final, yf):
    """argument fields and an aligned workspace of an SSD call"""
    b, L, H, P = x.shape
    G, Nst = B.shape[2], B.shape[3]
    fields = dict(batch=b, seqlen=L, nheads=H, headdim=P, dstate=Nst, ngroups=G, chunk=chunk,
                  state_group_size=state_group_size,
                  **_x_fields(x, x_group, x_scale, se_scale, se_log2_ratio),
                  dt=dt, dt_bias=dt_bias, dt_softplus=int(bool(dt_softplus)), A=A, D=D, z=z,
                  B=B, C=C, B_scale=B_scale, C_scale=C_scale, h0=h0, y=y, h_final=h_final,
                  status=status, max_segments=max_segments, dec_final=dec_final, **yf)
    ws = N.ssmq_ssd_workspace_size(**fields)
    _workspace(workspace, ws, x.device)
    if ws and workspace is None:
        workspace = torch.empty(ws + 256, dtype=torch.uint8, device=x.device)
    wptr = (workspace.data_ptr() + 255) // 256 * 256 if ws else None
    return fields, wptr, ws


def ssd_chunk_scan(x, dt, A, B, C, B_scale, C_scale, state_group_size, *, chunk=256,
                   x_group=None, x_scale=None, se_scale=0.0, se_log2_ratio=2, D=None, z=None,
                   dt_bias=None, dt_softplus=True, h0=None, y=None, h_final=None,
                   return_state=True, y_group=None, y_scale=None, y_q=None, want_y=True,
                   max_segments=0, dec_final=None, workspace=None, status=None):
    """Mamba-2 SSD chunked scan.  x (b, L, H, P) int8 / soft-edge uint8;
    dt (b, L, H) float16; B, C (b, L, G, N) int8.  Returns (y, h_final), or
    (y, h_final, y_q) with the int8 output (y_group over the H * P channels).
    max_segments = 1: one pass per sequence (byte-exact checkpoint / resume).
    dec_final: optional (b, H) float32 output, each sequence's total log2 decay."""
    b, L, H, P = x.shape
    Nst = B.shape[3]
    _dev_check(x, dt, A, B, C, B_scale, C_scale, x_group, x_scale, D, z, dt_bias, h0, dec_final)
    dv = x.device
    _ssd_inputs(x, dt, A, B, C, B_scale, C_scale, state_group_size, x_group, x_scale, D, z,
                dt_bias, h0)
    _out(h_final, "h_final", torch.float32, b * H * P * Nst, dv)
    _out(dec_final, "dec_final", torch.float32, b * H, dv)
    _status(status, dv)
    with _on(dv):
        y, y_q, yf = _y_fields((b, L, H, P), dv, y_group, y_scale, y_q, want_y, y, H * P)
        if h_final is None and return_state:
            h_final = torch.empty((b, H, P, Nst), dtype=torch.float32, device=dv)
        fields, wptr, ws = _ssd_call(x, dt, A, B, C, B_scale, C_scale, state_group_size, chunk,
                                     x_group, x_scale, se_scale, se_log2_ratio, D, z, dt_bias,
                                     dt_softplus, h0, y, h_final, max_segments, workspace,
                                     status, dec_final, yf)
        N.ssmq_ssd_chunk_scan_w8(workspace=wptr, ws_bytes=ws, **fields)
    return (y, h_final, y_q) if yf else (y, h_final)


def ssd_carry_in(x, dt, A, B, C, B_scale, C_scale, state_group_size, h_carry, y, *, chunk=256,
                 x_group=None, x_scale=None, se_scale=0.0, se_log2_ratio=2, D=None, z=None,
                 dt_bias=None, dt_softplus=True, h_final=None, workspace=None, status=None):
    """Adds the contribution of the start state h_carry (b, H, P, N) to the y
    (in place) and h_final (in place, if given) of an SSD call on the same
    inputs that started from a zero state."""
    _dev_check(x, dt, A, B, C, B_scale, C_scale, x_group, x_scale, D, z, dt_bias, h_carry, y,
               h_final)
    b, L, H, P = x.shape
    Nst = B.shape[3]
    dv = x.device
    _ssd_inputs(x, dt, A, B, C, B_scale, C_scale, state_group_size, x_group, x_scale, D, z,
                dt_bias, None)
    _out(y, "y", torch.float16, b * L * H * P, dv)
    _out(h_carry, "h_carry", torch.float32, b * H * P * Nst, dv)
    _out(h_final, "h_final", torch.float32, b * H * P * Nst, dv)
    _status(status, dv)
    with _on(dv):
        fields, wptr, ws = _ssd_call(x, dt, A, B, C, B_scale, C_scale, state_group_size, chunk,
                                     x_group, x_scale, se_scale, se_log2_ratio, D, z, dt_bias,
                                     dt_softplus, None, y, h_final, 0, workspace, status, None,
                                     {})
        N.ssmq_ssd_carry_in(h_carry, workspace=wptr, ws_bytes=ws, **fields)
    return y, h_final


def state_chain(h_ends, decs):
    """Fold of h <- exp2(dec_q) h + h_end_q over the parts q in order, from a
    zero state.  h_ends: sequence of equal-shape float32 tensors (units...,
    elems...) or one stacked tensor; decs likewise with one value per unit."""
    he = torch.stack(list(h_ends)) if not torch.is_tensor(h_ends) else h_ends
    dc = torch.stack(list(decs)) if not torch.is_tensor(decs) else decs
    he, dc = he.contiguous(), dc.contiguous()
    _dev_check(he, dc)
    n_parts = he.shape[0]
    units = dc[0].numel()
    elems = he[0].numel() // max(units, 1)
    _in(he, "h_ends", torch.float32, n_parts * units * elems, he.device)
    _in(dc, "decs", torch.float32, n_parts * units, he.device)
    with _on(he.device):
        out = torch.empty(he.shape[1:], dtype=torch.float32, device=he.device)
        N.ssmq_state_chain(he, dc, n_parts, units, elems, out)
    return out


def state_update(state, x, dt, A, B, C, B_scale, C_scale, state_group_size, *, x_group=None,
                 x_scale=None, se_scale=0.0, se_log2_ratio=2, D=None, z=None, dt_bias=None,
                 dt_softplus=True, y=None, status=None):
    """One decode step in place on ``state`` (b, H, P, N) fp32.  x (b, H, P);
    dt (b, H); B, C (b, G, N).  Returns y (b, H, P) float16."""
    b, H, P, Nst = state.shape
    G = B.shape[1]
    _dev_check(state, x, dt, A, B, C, B_scale, C_scale, x_group, x_scale, D, z, dt_bias)
    dv = state.device
    _x_in(x, x_group, x_scale, H * P, dv, codes_only=True)
    _in(x, "x", (torch.int8, torch.uint8), b * H * P, dv)
    _in(dt, "dt", torch.float16, b * H, dv)
    _in(z, "z", torch.float16, b * H * P, dv)
    for t, name in ((A, "A"), (D, "D"), (dt_bias, "dt_bias")):
        _in(t, name, torch.float32, H, dv)
    _bc_in(B, C, B_scale, C_scale, b * G * Nst, _n_scales(G, Nst, state_group_size), dv)
    _out(state, "state", torch.float32, b * H * P * Nst, dv)
    _out(y, "y", torch.float16, b * H * P, dv)
    _status(status, dv)
    with _on(dv):
        if y is None:
            y = torch.empty((b, H, P), dtype=torch.float16, device=dv)
        N.ssmq_state_update_w8(batch=b, nheads=H, headdim=P, dstate=Nst, ngroups=G,
                               state_group_size=state_group_size,
                               **_x_fields(x, x_group, x_scale, se_scale, se_log2_ratio),
                               dt=dt, dt_bias=dt_bias, dt_softplus=int(bool(dt_softplus)), A=A,
                               D=D, z=z, B=B, C=C, B_scale=B_scale, C_scale=C_scale,
                               state=state, y=y, status=status)
    return y


def selective_state_update(state, x, dt, A, B, C, B_scale, C_scale, state_group_size, *,
                           x_group=None, x_scale=None, se_scale=0.0, se_log2_ratio=2, D=None,
                           z=None, dt_bias=None, dt_softplus=True, y=None, status=None):
    """One Mamba-1 decode step in place on ``state`` (b, d, N) fp32.  x, dt, z
    (b, d); B, C (b, G, N); A (d, N).  Returns y (b, d) float16."""
    b, d, Nst = state.shape
    G = B.shape[1]
    _dev_check(state, x, dt, A, B, C, B_scale, C_scale, x_group, x_scale, D, z, dt_bias)
    dv = state.device
    _x_in(x, x_group, x_scale, d, dv, codes_only=True)
    _in(x, "x", (torch.int8, torch.uint8), b * d, dv)
    _in(dt, "dt", torch.float16, b * d, dv)
    _in(z, "z", torch.float16, b * d, dv)
    _in(A, "A", torch.float32, d * Nst, dv)
    _in(D, "D", torch.float32, d, dv)
    _in(dt_bias, "dt_bias", torch.float32, d, dv)
    _bc_in(B, C, B_scale, C_scale, b * G * Nst, _n_scales(G, Nst, state_group_size), dv)
    _out(state, "state", torch.float32, b * d * Nst, dv)
    _out(y, "y", torch.float16, b * d, dv)
    _status(status, dv)
    with _on(dv):
        if y is None:
            y = torch.empty((b, d), dtype=torch.float16, device=dv)
        N.ssmq_selective_state_update_w8(batch=b, dim=d, dstate=Nst, ngroups=G,
                                         state_group_size=state_group_size,
                                         **_x_fields(x, x_group, x_scale, se_scale,
                                                     se_log2_ratio),
                                         dt=dt, dt_bias=dt_bias,
                                         dt_softplus=int(bool(dt_softplus)), A=A, D=D, z=z, B=B,
                                         C=C, B_scale=B_scale, C_scale=C_scale, state=state, y=y,
                                         status=status)
    return y


# ---- calibration on the device ----------------------------------------------

def group_absmax(src, outer, mid, inner, group_of_mid, n_groups, *, out=None, status=None):
    """Exact max |v| per group over the finite elements (float32[n_groups])."""
    _dev_check(src, group_of_mid)
    dv = src.device
    _in(src, "src", _FP, outer * mid * inner, dv)
    _in(group_of_mid, "group_of_mid", torch.int32, mid, dv)
    _out(out, "out", torch.float32, n_groups, dv)
    _status(status, dv)
    with _on(dv):
        a = out if out is not None else torch.empty(n_groups, dtype=torch.float32, device=dv)
        N.ssmq_group_absmax(src, outer, mid, inner, group_of_mid, n_groups, a, status=status)
    return a


def cluster_by_absmax(absmax, k, *, status=None):
    """Sort-and-cluster on the device: (cluster id per channel int32, scales float32[k])."""
    _dev_check(absmax)
    _in(absmax, "absmax", torch.float32, None, absmax.device)
    _status(status, absmax.device)
    n = absmax.numel()
    with _on(absmax.device):
        cl = torch.empty(n, dtype=torch.int32, device=absmax.device)
        sc = torch.empty(k, dtype=torch.float32, device=absmax.device)
        N.ssmq_cluster_by_absmax(absmax, n, k, cl, sc, status=status)
    return cl, sc


def _pct_workspace(device, workspace):
    nb = N.ssmq_percentile_workspace_size()
    _workspace(workspace, nb, device)
    if workspace is None:
        workspace = torch.empty(nb + 256, dtype=torch.uint8, device=device)
    base = workspace.data_ptr()
    return (base + 255) // 256 * 256, nb


def _qlist(q):
    return [float(v) for v in (q if hasattr(q, "__len__") else [q])]


def percentile_abs(src, q, *, out=None, workspace=None):
    """Percentiles (linear interpolation) of |src| over its finite elements."""
    _dev_check(src)
    _in(src, "src", _FP, None, src.device)
    q = _qlist(q)
    _out(out, "out", torch.float32, len(q), src.device)
    with _on(src.device):
        o = out if out is not None else torch.empty(len(q), dtype=torch.float32,
                                                    device=src.device)
        wptr, nb = _pct_workspace(src.device, workspace)
        N.ssmq_percentile_abs(src, src.numel(), q, o, wptr, nb)
    return o


def softedge_calibrate(src, thresholds=None, *, q_lo=5.0, q_hi=99.9, alpha=1.0, workspace=None):
    """Soft-edge parameters {scale, lo, hi} (float32[3], updated in place):
    percentiles of |src|, blended into the running values when alpha < 1."""
    _dev_check(src)
    _in(src, "src", _FP, None, src.device)
    _out(thresholds, "thresholds", torch.float32, 3, src.device)
    with _on(src.device):
        thr = thresholds if thresholds is not None else torch.zeros(3, dtype=torch.float32,
                                                                      device=src.device)
        wptr, nb = _pct_workspace(src.device, workspace)
        N.ssmq_softedge_calibrate(src, src.numel(), q_lo, q_hi, alpha, thr, wptr, nb)
    return thr


# Allocation-free forms: the library's own static device scratch replaces the
# workspace, so a caller that may not allocate device memory (a CUDA graph
# being captured, an allocator-free serving loop) can still calibrate.  The
# out / thresholds tensors are the caller's.  Calls on one device share the
# scratch: do not let two overlap on the GPU.

def percentile_abs_noalloc(src, q, out):
    """percentile_abs into the caller's ``out`` (float32[len(q)]), with the
    library's static scratch; nothing is allocated."""
    _dev_check(src, out)
    _in(src, "src", _FP, None, src.device)
    q = _qlist(q)
    _out(out, "out", torch.float32, len(q), src.device)
    with _on(src.device):
        N.ssmq_percentile_abs_noalloc(src, src.numel(), q, out)
    return out


def softedge_calibrate_noalloc(src, thresholds, *, q_lo=5.0, q_hi=99.9, alpha=1.0):
    """softedge_calibrate on the caller's ``thresholds`` (float32[3], in
    place), with the library's static scratch; nothing is allocated."""
    _dev_check(src, thresholds)
    _in(src, "src", _FP, None, src.device)
    _out(thresholds, "thresholds", torch.float32, 3, src.device)
    with _on(src.device):
        N.ssmq_softedge_calibrate_noalloc(src, src.numel(), q_lo, q_hi, alpha, thresholds)
    return thresholds
