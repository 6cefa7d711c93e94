"""The C-ABI library on a CPU-only host: it loads, exports every entry point
declared in include/*.h, its argument structs have the layout the binding
assumes, and invalid arguments are rejected before any device call."""
import ctypes as C
import glob
import os
import re
import subprocess

import pytest

from quantized_state_space_b200 import _native as N
from quantized_state_space_b200 import build_native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build_native.build()
    return N.lib()


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(ssmq_[a-z0-9_]+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(L):
    declared = _declared()
    assert {"ssmq_quantize_groups", "ssmq_selective_scan_w8", "ssmq_ssd_chunk_scan_w8",
            "ssmq_state_update_w8", "ssmq_softedge_encode", "ssmq_softedge_decode"} <= declared
    out = subprocess.check_output(["nm", "-D", "--defined-only", N.LIB_PATH], text=True)
    exported = set(re.findall(r"\bT (ssmq_\w+)", out))
    assert declared <= exported, declared - exported
    assert declared <= set(N.SIGNATURES), declared - set(N.SIGNATURES)


STRUCTS = ((N.ScanArgs, "ssmq_scan_args"), (N.SSDArgs, "ssmq_ssd_args"),
           (N.DecodeArgs, "ssmq_decode_args"), (N.M1DecodeArgs, "ssmq_m1_decode_args"),
           (N.ConvArgs, "ssmq_conv_args"))


def test_struct_layout_matches_header(tmp_path):
    prog = ["#include <stdio.h>", "#include <stddef.h>", '#include "ssmq.h"', "int main(void){"]
    for cls, cname in STRUCTS:
        prog.append('printf("%s %%zu\\n", sizeof(%s));' % (cname, cname))
        for f, _ in cls._fields_:
            prog.append('printf("%s.%s %%zu\\n", offsetof(%s, %s));' % (cname, f, cname, f))
    prog.append("return 0;}")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(prog))
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)])
    got = dict(line.split() for line in subprocess.check_output([str(exe)], text=True).splitlines())
    for cls, cname in STRUCTS:
        assert int(got[cname]) == C.sizeof(cls), cname
        for f, _ in cls._fields_:
            assert int(got["%s.%s" % (cname, f)]) == getattr(cls, f).offset, (cname, f)


FAKE = 0x10000  # an aligned, never-dereferenced address for validation tests


def _status_of(fn, *a):
    return getattr(N.lib(), fn)(*a)


def test_quantize_validation(L):
    Q = L.ssmq_quantize_groups
    assert Q(FAKE, 5, 1, 1, 16, FAKE, 1, 0, FAKE, FAKE, None, None) == N.ERR_INVALID_ARG  # dtype
    assert Q(FAKE, 1, 1, 1, 16, FAKE, 1, 7, FAKE, FAKE, None, None) == N.ERR_INVALID_ARG  # mode
    assert Q(FAKE, 1, -1, 1, 16, FAKE, 1, 0, FAKE, FAKE, None, None) == N.ERR_INVALID_ARG
    assert Q(FAKE, 1, 1, 1, 16, FAKE, 0, 0, FAKE, FAKE, None, None) == N.ERR_INVALID_ARG
    assert Q(None, 1, 1, 1, 16, FAKE, 1, 0, FAKE, FAKE, None, None) == N.ERR_INVALID_ARG
    assert "NULL" in N.ssmq_last_error()
    assert Q(FAKE + 2, 1, 1, 1, 16, FAKE, 1, 0, FAKE, FAKE, None, None) == N.ERR_ALIGNMENT
    # empty static problem: nothing to do, no launch
    assert Q(None, 1, 0, 5, 16, None, 1, 0, FAKE, None, None, None) == N.OK


def test_softedge_validation(L):
    E = L.ssmq_softedge_encode
    assert E(FAKE, 1, 16, 1.0, 2.0, 1.0, 2, FAKE, None, None) == N.ERR_INVALID_ARG  # L > H
    assert "thr_lo" in N.ssmq_last_error()
    assert E(FAKE, 1, 16, 1.0, 0.5, 1.0, 9, FAKE, None, None) == N.ERR_INVALID_ARG
    assert E(FAKE, 1, 16, 1.0, 0.5, 1.0, 2, FAKE + 8, None, None) == N.ERR_ALIGNMENT
    D = L.ssmq_softedge_decode
    assert D(None, 16, 1.0, 2, FAKE, None) == N.ERR_INVALID_ARG
    assert D(FAKE, -1, 1.0, 2, FAKE, None) == N.ERR_INVALID_ARG


def _scan_args(**kw):
    f = dict(batch=2, seqlen=64, dim=32, dstate=16, ngroups=1, state_group_size=4,
             x_format=N.X_INT8_GROUP, x=FAKE, x_group=FAKE, x_scale=FAKE, n_x_groups=4,
             dt=FAKE, A=FAKE, B=FAKE, C=FAKE, B_scale=FAKE, C_scale=FAKE, y=FAKE,
             dt_softplus=1)
    f.update(kw)
    return N._fill(N.ScanArgs, f)


def test_scan_validation(L):
    S = lambda **kw: L.ssmq_selective_scan_w8(C.byref(_scan_args(**kw)), None)
    assert S(dstate=12) == N.ERR_UNSUPPORTED
    assert S(dstate=128) == N.ERR_UNSUPPORTED
    assert S(ngroups=3) == N.ERR_INVALID_ARG
    assert S(state_group_size=3) == N.ERR_INVALID_ARG
    assert S(x_format=5) == N.ERR_INVALID_ARG
    assert S(x_group=None) == N.ERR_INVALID_ARG
    assert S(n_x_groups=0) == N.ERR_INVALID_ARG
    assert S(dt=None) == N.ERR_INVALID_ARG
    assert S(y=FAKE + 4) == N.ERR_ALIGNMENT
    assert S(x_format=N.X_SOFTEDGE, x_group=None, x_scale=None, se_log2_ratio=12) == N.ERR_INVALID_ARG
    # binary16 x encoded in the kernel: group form needs the cluster map, the
    # soft-edge form ordered thresholds (as ssmq_softedge_encode)
    assert S(x_format=N.X_F16_GROUP, x_group=None) == N.ERR_INVALID_ARG
    assert S(x_format=N.X_F16_SOFTEDGE, x_group=None, x_scale=None, se_lo=2.0,
             se_hi=1.0) == N.ERR_INVALID_ARG
    assert S(x_format=N.X_F16_SOFTEDGE, x_group=None, x_scale=None, se_lo=float("nan"),
             se_hi=1.0) == N.ERR_INVALID_ARG
    assert S(x_format=4) == N.ERR_INVALID_ARG
    # int8 y: needs its cluster map; y may be dropped only when y_q is given
    assert S(y_q=FAKE, y_group=None, y_scale=FAKE, n_y_groups=2) == N.ERR_INVALID_ARG
    assert S(y_q=FAKE, y_group=FAKE, y_scale=FAKE, n_y_groups=0) == N.ERR_INVALID_ARG
    assert S(y_q=FAKE + 8, y_group=FAKE, y_scale=FAKE, n_y_groups=2) == N.ERR_ALIGNMENT
    assert S(y=None) == N.ERR_INVALID_ARG
    assert S(batch=0) == N.OK
    assert L.ssmq_selective_scan_w8(None, None) == N.ERR_INVALID_ARG


def test_scan_time_segments_rule(L):
    """Segments of whole 32-step chunks; one pass without binary16 y, with
    int8 y, below 64 steps or beyond 65535 (batch x segments) rows; the
    workspace holds every segment's fp32 (d, N) state per batch row."""
    K = lambda **kw: L.ssmq_scan_time_segments(C.byref(_scan_args(**kw)))
    W = lambda **kw: L.ssmq_scan_workspace_size(C.byref(_scan_args(**kw)))
    a = dict(batch=2, seqlen=2048, dim=64, dstate=16)
    assert K(**a) == 1 and W(**a) == 0
    assert K(time_segments=0, **a) == 1
    assert K(time_segments=2, **a) == 2 and W(time_segments=2, **a) == 2 * 2 * 64 * 16 * 4
    assert K(time_segments=4, **a) == 4
    assert K(time_segments=3, batch=2, seqlen=100, dim=64, dstate=16) == 2  # 34 -> 64 steps
    assert K(time_segments=8, batch=2, seqlen=64, dim=64, dstate=16) == 2   # whole chunks
    assert K(time_segments=2, batch=2, seqlen=63, dim=64, dstate=16) == 1
    assert K(time_segments=2, y=None, y_q=FAKE, y_group=FAKE, y_scale=FAKE, n_y_groups=1,
             **a) == 1
    assert K(time_segments=2, batch=40000, seqlen=2048, dim=64, dstate=16) == 1
    assert L.ssmq_scan_time_segments(None) == 0 and L.ssmq_scan_workspace_size(None) == 0


def test_scan_time_segments_validation(L):
    S = lambda **kw: L.ssmq_selective_scan_w8(C.byref(_scan_args(**kw)), None)
    a = dict(time_segments=2, seqlen=2048)
    nb = L.ssmq_scan_workspace_size(C.byref(_scan_args(**a)))
    assert nb > 0
    assert S(**a) == N.ERR_INVALID_ARG                                   # no workspace
    assert S(workspace=FAKE, workspace_bytes=nb - 4, **a) == N.ERR_INVALID_ARG
    assert S(workspace=FAKE + 8, workspace_bytes=nb, **a) == N.ERR_ALIGNMENT
    # one pass: the workspace is not looked at
    assert S(batch=0, **a) == N.OK


def test_scan_carry_in_validation(L):
    K = lambda h=FAKE, **kw: L.ssmq_selective_scan_carry_in(C.byref(_scan_args(**kw)), h, None)
    assert K(h=None) == N.ERR_INVALID_ARG
    assert K(dstate=12) == N.ERR_UNSUPPORTED
    assert K(y=None) == N.ERR_INVALID_ARG
    assert K(C_scale=None) == N.ERR_INVALID_ARG
    assert K(h=FAKE + 4) == N.ERR_ALIGNMENT
    assert K(batch=0, h=None) == N.OK
    assert L.ssmq_selective_scan_carry_in(None, FAKE, None) == N.ERR_INVALID_ARG
    # a call with log2 decays keeps one pass
    assert L.ssmq_scan_time_segments(C.byref(_scan_args(time_segments=4, seqlen=2048,
                                                        dec_final=FAKE))) == 1


def _ssd_args(**kw):
    f = dict(batch=1, seqlen=512, nheads=8, headdim=64, dstate=128, ngroups=1, chunk=256,
             state_group_size=8, x_format=N.X_INT8_GROUP, x=FAKE, x_group=FAKE, x_scale=FAKE,
             n_x_groups=2, dt=FAKE, A=FAKE, B=FAKE, C=FAKE, B_scale=FAKE, C_scale=FAKE, y=FAKE,
             dt_softplus=1)
    f.update(kw)
    return N._fill(N.SSDArgs, f)


def test_ssd_validation(L):
    S = lambda ws=None, nb=0, **kw: L.ssmq_ssd_chunk_scan_w8(C.byref(_ssd_args(**kw)), ws, nb, None)
    assert S(headdim=32) == N.ERR_UNSUPPORTED
    assert S(chunk=100) == N.ERR_UNSUPPORTED
    assert S(ngroups=3) == N.ERR_INVALID_ARG
    assert S(x=None) == N.ERR_INVALID_ARG
    assert S(x_format=N.X_F16_GROUP) == N.ERR_UNSUPPORTED  # Mamba-1 scan only
    assert S(y=None) == N.ERR_INVALID_ARG
    assert S(y_q=FAKE, y_group=None, y_scale=FAKE, n_y_groups=2) == N.ERR_INVALID_ARG
    need = L.ssmq_ssd_workspace_size(C.byref(_ssd_args()))
    if need:
        assert S(ws=None, nb=0) == N.ERR_INVALID_ARG
        assert S(ws=FAKE + 16, nb=need) == N.ERR_ALIGNMENT


def test_quantize_batch_validation(L):
    J = N.QuantJob
    ok = dict(src=FAKE, dtype=N.F16, outer=2, mid=4, inner=16, group_of_mid=FAKE, n_groups=2,
              scales=FAKE, q_out=FAKE)

    def S(n=1, **kw):
        arr = (J * max(n, 1))()
        for i in range(max(n, 1)):
            arr[i] = N._fill(J, dict(ok, **kw))
        return L.ssmq_quantize_groups_batch(arr, n, None, None)

    assert L.ssmq_quantize_groups_batch(None, 1, None, None) == N.ERR_INVALID_ARG
    assert S(n=0) == N.ERR_INVALID_ARG
    assert S(n=9) == N.ERR_INVALID_ARG
    assert S(dtype=7) == N.ERR_INVALID_ARG
    assert S(n_groups=0) == N.ERR_INVALID_ARG
    assert S(scales=None) == N.ERR_INVALID_ARG
    assert S(outer=-1) == N.ERR_INVALID_ARG
    assert S(q_out=None) == N.ERR_INVALID_ARG
    assert S(src=FAKE + 8) == N.ERR_ALIGNMENT
    assert S(outer=1 << 40, mid=1 << 20, inner=1 << 10) == N.ERR_INVALID_ARG


def test_sequence_sharding_validation(L):
    assert L.ssmq_state_chain(FAKE, FAKE, 0, 4, 8, FAKE, None) == N.ERR_INVALID_ARG
    assert L.ssmq_state_chain(FAKE, FAKE, 2, -1, 8, FAKE, None) == N.ERR_INVALID_ARG
    assert L.ssmq_state_chain(None, FAKE, 2, 4, 8, FAKE, None) == N.ERR_INVALID_ARG
    assert L.ssmq_state_chain(FAKE, FAKE, 2, 1 << 40, 1 << 30, FAKE, None) == N.ERR_INVALID_ARG
    assert L.ssmq_state_chain(None, None, 2, 0, 8, None, None) == N.OK  # nothing to do
    def S(hc=FAKE, **kw):
        a = _ssd_args(**kw)  # kept alive across the call
        return L.ssmq_ssd_carry_in(C.addressof(a), hc, FAKE, 1 << 40, None)

    assert S(hc=None) == N.ERR_INVALID_ARG
    assert S(hc=FAKE + 4) == N.ERR_ALIGNMENT
    assert S(y=None, y_q=FAKE, y_group=FAKE, y_scale=FAKE, n_y_groups=1) == N.ERR_INVALID_ARG
    assert S(headdim=32) == N.ERR_UNSUPPORTED
    assert L.ssmq_ssd_carry_in(None, FAKE, FAKE, 0, None) == N.ERR_INVALID_ARG


def test_ssd_workspace_size_rule(L):
    """Operand blocks (64 KB per batch, group and 128-step tile), plus, when
    sequences may be cut into segments, one fp32 (P, N) state and one decay
    per segment slot: min(256, sequences x min(cap, tiles)) slots."""
    W = lambda **kw: L.ssmq_ssd_workspace_size(C.byref(_ssd_args(**kw)))
    ops = lambda b, g, L_: b * g * ((L_ + 127) // 128) * 65536
    slot = 64 * 128 * 4 + 4
    assert W(max_segments=1) == ops(1, 1, 512)
    assert W() == ops(1, 1, 512) + 8 * 4 * slot                 # 8 sequences, 4 tiles
    assert W(seqlen=100) == ops(1, 1, 100)                      # one tile: never cut
    assert W(max_segments=3) == ops(1, 1, 512) + 8 * 3 * slot
    assert W(seqlen=128 * 100, batch=2) == ops(2, 1, 128 * 100) + 256 * slot
    assert W(seqlen=128 * 100, nheads=1) == ops(1, 1, 128 * 100) + 32 * slot
    assert W(y_q=FAKE, y_group=FAKE, y_scale=FAKE, n_y_groups=1) == ops(1, 1, 512)
    assert W(y=None) == ops(1, 1, 512)
    assert W(seqlen=0) == 0


def _dec_args(**kw):
    f = dict(batch=4, nheads=8, headdim=64, dstate=128, ngroups=2, state_group_size=8,
             x_format=N.X_INT8_GROUP, x=FAKE, x_group=FAKE, x_scale=FAKE, n_x_groups=2, dt=FAKE,
             A=FAKE, B=FAKE, C=FAKE, B_scale=FAKE, C_scale=FAKE, state=FAKE, y=FAKE,
             dt_softplus=1)
    f.update(kw)
    return N._fill(N.DecodeArgs, f)


def test_decode_validation(L):
    S = lambda **kw: L.ssmq_state_update_w8(C.byref(_dec_args(**kw)), None)
    assert S(dstate=96) == N.ERR_UNSUPPORTED
    assert S(ngroups=3) == N.ERR_INVALID_ARG
    assert S(state=None) == N.ERR_INVALID_ARG
    assert S(state=FAKE + 4) == N.ERR_ALIGNMENT
    assert S(x_format=N.X_F16_SOFTEDGE) == N.ERR_UNSUPPORTED  # Mamba-1 scan only
    assert S(batch=0) == N.OK


def test_fault_injection_hook(L, monkeypatch):
    """SSMQ_FAULT_INJECT makes the named entry point report a launch failure
    after validation, without touching the device."""
    monkeypatch.setenv("SSMQ_FAULT_INJECT", "ssmq_selective_scan_w8")
    assert L.ssmq_selective_scan_w8(C.byref(_scan_args()), None) == N.ERR_CUDA
    assert "injected" in N.ssmq_last_error()
    with pytest.raises(N.SSMQError) as ei:
        N.ssmq_selective_scan_w8(stream=0, **{k: getattr(_scan_args(), k)
                                               for k, _ in N.ScanArgs._fields_})
    assert ei.value.status == N.ERR_CUDA
    # validation still runs first
    assert L.ssmq_selective_scan_w8(C.byref(_scan_args(dt=None)), None) == N.ERR_INVALID_ARG
    monkeypatch.setenv("SSMQ_FAULT_INJECT", "all")
    assert L.ssmq_state_update_w8(C.byref(_dec_args()), None) == N.ERR_CUDA
    assert L.ssmq_quantize_groups(FAKE, 1, 1, 1, 16, FAKE, 1, 0, FAKE, FAKE, None, None) == N.ERR_CUDA


def test_version(L):
    assert N.ssmq_version() >= 100


def test_probe_validation(L):
    n = C.c_int64(-1)
    assert L.ssmq_probe_ex2(0, FAKE, C.byref(n), None) == N.ERR_INVALID_ARG
    assert L.ssmq_probe_ex2(16, None, C.byref(n), None) == N.ERR_INVALID_ARG
    assert L.ssmq_probe_ex2(16, FAKE, None, None) == N.ERR_INVALID_ARG
    assert L.ssmq_probe_ex2(16, FAKE + 4, C.byref(n), None) == N.ERR_ALIGNMENT
    assert n.value == -1  # nothing written on a rejected call


def test_m1_decode_validation(L):
    f = dict(batch=4, dim=32, dstate=16, ngroups=1, state_group_size=4, x_format=N.X_INT8_GROUP,
             x=FAKE, x_group=FAKE, x_scale=FAKE, n_x_groups=2, dt=FAKE, A=FAKE, B=FAKE, C=FAKE,
             B_scale=FAKE, C_scale=FAKE, state=FAKE, y=FAKE, dt_softplus=1)

    def S(**kw):
        g = dict(f)
        g.update(kw)
        return L.ssmq_selective_state_update_w8(C.byref(N._fill(N.M1DecodeArgs, g)), None)
    assert S(dstate=12) == N.ERR_UNSUPPORTED
    assert S(ngroups=3) == N.ERR_INVALID_ARG
    assert S(A=None) == N.ERR_INVALID_ARG
    assert S(A=FAKE + 4) == N.ERR_ALIGNMENT
    assert S(batch=0) == N.OK


def test_calibration_validation(L):
    """Device calibration calls reject bad arguments before any launch."""
    F = N.F16
    assert L.ssmq_group_absmax(FAKE, 7, 2, 3, 4, FAKE, 3, FAKE, None, None) == N.ERR_INVALID_ARG
    assert L.ssmq_group_absmax(FAKE, F, 2, 3, 4, FAKE, 0, FAKE, None, None) == N.ERR_INVALID_ARG
    assert L.ssmq_group_absmax(FAKE + 2, F, 2, 3, 4, FAKE, 3, FAKE, None, None) == N.ERR_ALIGNMENT
    assert L.ssmq_cluster_by_absmax(FAKE, 10, 11, FAKE, FAKE, None, None) == N.ERR_INVALID_ARG
    assert L.ssmq_cluster_by_absmax(FAKE, 10, 0, FAKE, FAKE, None, None) == N.ERR_INVALID_ARG
    assert L.ssmq_cluster_by_absmax(FAKE, 70000, 8, FAKE, FAKE, None, None) == N.ERR_UNSUPPORTED
    nb = L.ssmq_percentile_workspace_size()
    assert nb >= 32768 * 4
    q = (C.c_double * 2)(5.0, 99.9)
    P = lambda **kw: L.ssmq_percentile_abs(kw.get("src", FAKE), F, 100, kw.get("q", q),
                                           kw.get("nq", 2), FAKE, kw.get("ws", FAKE),
                                           kw.get("nb", nb), None)
    assert P(nb=nb - 1) == N.ERR_INVALID_ARG
    assert P(ws=FAKE + 16) == N.ERR_ALIGNMENT
    assert P(nq=0) == N.ERR_INVALID_ARG
    assert P(q=(C.c_double * 2)(5.0, 100.5)) == N.ERR_INVALID_ARG
    assert P(src=None) == N.ERR_INVALID_ARG
    S = lambda lo, hi, a: L.ssmq_softedge_calibrate(FAKE, F, 100, lo, hi, a, FAKE, FAKE, nb, None)
    assert S(5.0, 99.9, 0.0) == N.ERR_INVALID_ARG
    assert S(5.0, 99.9, 1.5) == N.ERR_INVALID_ARG
    assert S(99.9, 5.0, 0.1) == N.ERR_INVALID_ARG


def _conv_args(**kw):
    a = N.ConvArgs(batch=2, seqlen=32, dim=8, width=4, x=FAKE, weight=FAKE, bias=None,
                   x_prev=None, out_format=N.X_INT8_GROUP, x_group=FAKE, x_scale=FAKE,
                   n_x_groups=2, se_scale=1.0, se_lo=0.1, se_hi=5.0, se_log2_ratio=2,
                   codes=FAKE, u=None, x_prev_out=None, status=None)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_conv_validation(L):
    S = lambda **kw: L.ssmq_conv_silu_quantize(C.byref(_conv_args(**kw)), None)
    assert L.ssmq_conv_silu_quantize(None, None) == N.ERR_INVALID_ARG
    assert S(width=0) == N.ERR_INVALID_ARG
    assert S(width=5) == N.ERR_INVALID_ARG
    assert S(seqlen=-1) == N.ERR_INVALID_ARG
    assert S(out_format=N.X_F16_GROUP) == N.ERR_INVALID_ARG
    assert S(x_group=None) == N.ERR_INVALID_ARG
    assert S(n_x_groups=0) == N.ERR_INVALID_ARG
    assert S(out_format=N.X_SOFTEDGE, se_lo=6.0, se_hi=5.0) == N.ERR_INVALID_ARG
    assert S(out_format=N.X_SOFTEDGE, se_log2_ratio=9) == N.ERR_INVALID_ARG
    assert S(x=None) == N.ERR_INVALID_ARG
    assert S(codes=None) == N.ERR_INVALID_ARG
    assert S(x=FAKE + 2) == N.ERR_ALIGNMENT
    assert S(u=FAKE + 8) == N.ERR_ALIGNMENT
    # the two conv states may not overlap (2 * 8 * 3 binary16 = 96 bytes each)
    assert S(x_prev=FAKE, x_prev_out=FAKE + 64) == N.ERR_INVALID_ARG
    assert S(batch=0, x=None, codes=None, x_prev=FAKE, x_prev_out=FAKE + 96,
             x_group=None) == N.ERR_INVALID_ARG  # group map still required
