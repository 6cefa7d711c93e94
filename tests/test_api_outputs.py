"""The Python front end checks every tensor that the caller supplies to a
call, read or written -- device, contiguity, dtype, element count -- since
the C library sees only pointers.  Run on the CPU: the native
calls are replaced by a recorder and the CUDA-device requirement is lifted,
so only the front end's own checks decide."""
import pytest
import torch

from quantized_state_space_b200 import _native as real_native
from quantized_state_space_b200 import api


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if name == "ssmq_ssd_workspace_size":
            return lambda **kw: 4096
        if name == "ssmq_percentile_workspace_size":
            return lambda: 1024
        if name == "ssmq_scan_workspace_size":
            return lambda **kw: 512 if kw.get("time_segments", 1) > 1 else 0
        if name.startswith("ssmq_"):
            return lambda *a, **kw: self.calls.append(name)
        return getattr(real_native, name)


@pytest.fixture()
def rec(monkeypatch):
    r = _Recorder()
    monkeypatch.setattr(api, "N", r)
    monkeypatch.setattr(api, "_dev_check", lambda *ts: None)
    return r


def E(*shape, dtype=torch.float32, device="cpu"):
    return torch.empty(shape, dtype=dtype, device=device)


def _bad(fn, **kw):
    with pytest.raises(ValueError):
        fn(**kw)


def test_quantizer_outputs(rec):
    src, g, s = E(2, 3, 8, dtype=torch.float16), E(3, dtype=torch.int32), E(2)
    call = lambda **kw: api.quantize_groups(src, 2, 3, 8, g, 2, scales=s, **kw)
    call(out=E(48, dtype=torch.int8), status=E(1, dtype=torch.int32))
    _bad(call, out=E(47, dtype=torch.int8))
    _bad(call, out=E(48, dtype=torch.uint8))
    _bad(call, out=E(48, dtype=torch.int8, device="meta"))
    _bad(call, out=E(8, 6, dtype=torch.int8).t())
    _bad(call, status=E(1, dtype=torch.int16))
    _bad(call, status=E(0, dtype=torch.int32))
    job = lambda out: [(src, 2, 3, 8, g, 2, s, out)]
    api.quantize_groups_batch(job(E(48, dtype=torch.int8)))
    _bad(lambda **kw: api.quantize_groups_batch(job(E(40, dtype=torch.int8))))
    api.softedge_encode(src, 1.0, 0.1, 5.0, out=E(48, dtype=torch.uint8))
    _bad(lambda: api.softedge_encode(src, 1.0, 0.1, 5.0, out=E(48, dtype=torch.int8)))
    codes = E(48, dtype=torch.uint8)
    api.softedge_decode(codes, 1.0, out=E(48))
    _bad(lambda: api.softedge_decode(codes, 1.0, out=E(48, dtype=torch.float16)))
    assert rec.calls.count("ssmq_quantize_groups") == 1


def test_scan_outputs(rec):
    b, d, L, G, N = 2, 8, 5, 1, 16
    x, dt = E(b, d, L, dtype=torch.int8), E(b, d, L, dtype=torch.float16)
    Bq = E(b, G, N, L, dtype=torch.int8)
    args = (x, dt, E(d, N), Bq, Bq, E(4), E(4), 4)
    kw = dict(x_group=E(d, dtype=torch.int32), x_scale=E(2))
    api.selective_scan(*args, y=E(b, d, L, dtype=torch.float16), h_final=E(b, d, N), **kw)
    _bad(lambda: api.selective_scan(*args, y=E(b, d, L), **kw))
    _bad(lambda: api.selective_scan(*args, h_final=E(b, d, N - 1), **kw))
    _bad(lambda: api.selective_scan(*args, y_group=E(d, dtype=torch.int32), y_scale=E(2),
                                    y_q=E(b, d, L, dtype=torch.uint8), **kw))
    dec_args = (E(b, d, dtype=torch.int8), E(b, d, dtype=torch.float16), E(d, N),
                E(b, G, N, dtype=torch.int8), E(b, G, N, dtype=torch.int8), E(4), E(4), 4)
    api.selective_state_update(E(b, d, N), *dec_args, y=E(b, d, dtype=torch.float16), **kw)
    _bad(lambda: api.selective_state_update(E(b, d, N, dtype=torch.float64), *dec_args, **kw))
    _bad(lambda: api.selective_state_update(E(b, d, N), *dec_args, y=E(b, d + 1,
                                                                       dtype=torch.float16), **kw))


def test_ssd_outputs(rec):
    b, L, H, P, G, N = 1, 300, 2, 64, 1, 128
    x, dt = E(b, L, H, P, dtype=torch.int8), E(b, L, H, dtype=torch.float16)
    Bq = E(b, L, G, N, dtype=torch.int8)
    args = (x, dt, E(H), Bq, Bq, E(16), E(16), 8)
    kw = dict(x_group=E(H * P, dtype=torch.int32), x_scale=E(2))
    y, hf, dec = E(b, L, H, P, dtype=torch.float16), E(b, H, P, N), E(b, H)
    api.ssd_chunk_scan(*args, y=y, h_final=hf, dec_final=dec,
                       workspace=E(4096 + 255, dtype=torch.uint8), **kw)
    _bad(lambda: api.ssd_chunk_scan(*args, workspace=E(4096, dtype=torch.uint8), **kw))
    _bad(lambda: api.ssd_chunk_scan(*args, workspace=E(8192), **kw))
    _bad(lambda: api.ssd_chunk_scan(*args, dec_final=E(b, H + 1), **kw))
    _bad(lambda: api.ssd_chunk_scan(*args, h_final=E(b, H, N, P, dtype=torch.float16), **kw))
    api.ssd_carry_in(*args, E(b, H, P, N), y, h_final=hf, **kw)
    _bad(lambda: api.ssd_carry_in(*args, E(b, H, P, N - 8), y, **kw))
    _bad(lambda: api.ssd_carry_in(*args, E(b, H, P, N), E(b, L - 1, H, P, dtype=torch.float16),
                                  **kw))
    x0 = E(b, 0, H, P, dtype=torch.int8)  # an empty sequence: y has no elements
    api.ssd_carry_in(x0, E(b, 0, H, dtype=torch.float16), E(H), E(b, 0, G, N, dtype=torch.int8),
                     E(b, 0, G, N, dtype=torch.int8), E(16), E(16), 8, E(b, H, P, N),
                     E(b, 0, H, P, dtype=torch.float16), h_final=hf, **kw)
    st = E(2, H, P, N)
    api.state_update(st, E(2, H, P, dtype=torch.int8), E(2, H, dtype=torch.float16), E(H),
                     E(2, G, N, dtype=torch.int8), E(2, G, N, dtype=torch.int8), E(16), E(16), 8,
                     y=E(2, H, P, dtype=torch.float16), **kw)
    _bad(lambda: api.state_update(st, E(2, H, P, dtype=torch.int8), E(2, H, dtype=torch.float16),
                                  E(H), E(2, G, N, dtype=torch.int8), E(2, G, N, dtype=torch.int8),
                                  E(16), E(16), 8, y=E(2, H, P), **kw))


def test_calibration_outputs(rec):
    src = E(4, 6, dtype=torch.float16)
    api.group_absmax(src, 1, 4, 6, E(4, dtype=torch.int32), 4, out=E(4))
    _bad(lambda: api.group_absmax(src, 1, 4, 6, E(4, dtype=torch.int32), 4, out=E(3)))
    api.percentile_abs(src, [5.0, 99.9], out=E(2), workspace=E(1024 + 255, dtype=torch.uint8))
    _bad(lambda: api.percentile_abs(src, [5.0, 99.9], out=E(3)))
    _bad(lambda: api.percentile_abs(src, 5.0, workspace=E(1024, dtype=torch.uint8)))
    api.softedge_calibrate(src, E(3))
    _bad(lambda: api.softedge_calibrate(src, E(3, dtype=torch.float64)))


def test_scan_inputs(rec):
    """Every tensor a call reads is checked too: a short or mistyped input,
    or one on another device, would be read past its end or across devices."""
    b, d, L, G, N = 2, 8, 5, 1, 16
    good = dict(x=E(b, d, L, dtype=torch.int8), dt=E(b, d, L, dtype=torch.float16), A=E(d, N),
                B=E(b, G, N, L, dtype=torch.int8), C=E(b, G, N, L, dtype=torch.int8),
                B_scale=E(4), C_scale=E(4))
    kw = dict(x_group=E(d, dtype=torch.int32), x_scale=E(2), z=E(b, d, L, dtype=torch.float16),
              h0=E(b, d, N), D=E(d), dt_bias=E(d))

    def call(**over):
        a = dict(good, **{k: v for k, v in over.items() if k in good})
        k2 = dict(kw, **{k: v for k, v in over.items() if k not in good})
        return api.selective_scan(a["x"], a["dt"], a["A"], a["B"], a["C"], a["B_scale"],
                                  a["C_scale"], 4, **k2)

    call()
    # binary16 x soft-edge encoded in the scan: no cluster map needed
    call(x=E(b, d, L, dtype=torch.float16), x_group=None, x_scale=None, se_scale=1.0,
         se_lo=0.1, se_hi=5.0)
    _bad(call, x=E(b, d, L, dtype=torch.float16), x_group=None, x_scale=None)
    for bad in (dict(h0=E(b, d, N - 1)), dict(h0=E(b, d, N, dtype=torch.float16)),
                dict(dt=E(b, d, L - 1, dtype=torch.float16)), dict(dt=E(b, d, L)),
                dict(z=E(b, d, L - 1, dtype=torch.float16)),
                dict(C=E(b, G, N, L - 1, dtype=torch.int8)), dict(B=E(b, G, N, L, dtype=torch.uint8)),
                dict(C_scale=E(3)), dict(B_scale=E(4, dtype=torch.float64)),
                dict(A=E(d, N - 1)), dict(D=E(d + 1)), dict(dt_bias=E(d - 1)),
                dict(x_group=E(d - 1, dtype=torch.int32)), dict(x_group=E(d, dtype=torch.int64)),
                dict(x=E(b, d, L, dtype=torch.float32)),
                dict(h0=E(b, d, N, device="meta")), dict(A=E(d, N, device="meta"))):
        _bad(call, **bad)
    assert rec.calls.count("ssmq_selective_scan_w8") == 2


def test_ssd_and_decode_inputs(rec):
    b, L, H, P, G, N = 1, 300, 2, 64, 1, 128
    x, dt = E(b, L, H, P, dtype=torch.int8), E(b, L, H, dtype=torch.float16)
    Bq = E(b, L, G, N, dtype=torch.int8)
    kw = dict(x_group=E(H * P, dtype=torch.int32), x_scale=E(2))
    api.ssd_chunk_scan(x, dt, E(H), Bq, Bq, E(16), E(16), 8, h0=E(b, H, P, N), **kw)
    _bad(lambda: api.ssd_chunk_scan(x, dt, E(H), Bq, Bq, E(16), E(16), 8, h0=E(b, H, P, N - 1),
                                    **kw))
    _bad(lambda: api.ssd_chunk_scan(x, E(b, L - 1, H, dtype=torch.float16), E(H), Bq, Bq, E(16),
                                    E(16), 8, **kw))
    _bad(lambda: api.ssd_chunk_scan(x, dt, E(H), Bq, E(b, L, G, N - 1, dtype=torch.int8), E(16),
                                    E(16), 8, **kw))
    _bad(lambda: api.ssd_chunk_scan(x, dt, E(H), Bq, Bq, E(16), E(15), 8, **kw))
    _bad(lambda: api.ssd_chunk_scan(x, dt, E(H), Bq, Bq, E(16), E(16), 8,
                                    z=E(b, L, H, P - 1, dtype=torch.float16), **kw))
    _bad(lambda: api.ssd_chunk_scan(x, dt, E(H, device="meta"), Bq, Bq, E(16), E(16), 8, **kw))
    _bad(lambda: api.ssd_chunk_scan(x.to(torch.float16), dt, E(H), Bq, Bq, E(16), E(16), 8, **kw))
    st = E(2, H, P, N)
    dargs = lambda xx, dtt, BB: (st, xx, dtt, E(H), BB, BB, E(16), E(16), 8)
    good = (E(2, H, P, dtype=torch.int8), E(2, H, dtype=torch.float16),
            E(2, G, N, dtype=torch.int8))
    api.state_update(*dargs(*good), **kw)
    _bad(lambda: api.state_update(*dargs(E(2, H, P - 1, dtype=torch.int8), *good[1:]), **kw))
    _bad(lambda: api.state_update(*dargs(good[0], E(2, H + 1, dtype=torch.float16), good[2]),
                                  **kw))
    _bad(lambda: api.state_update(*dargs(*good[:2], E(2, G, N - 8, dtype=torch.int8)), **kw))


def test_quantizer_and_calibration_inputs(rec):
    src, g, s = E(2, 3, 8, dtype=torch.float16), E(3, dtype=torch.int32), E(2)
    _bad(lambda: api.quantize_groups(src, 2, 3, 8, E(2, dtype=torch.int32), 2, scales=s))
    _bad(lambda: api.quantize_groups(src, 2, 3, 8, g, 2, scales=E(1)))
    _bad(lambda: api.quantize_groups(src, 2, 3, 9, g, 2, scales=s))
    _bad(lambda: api.quantize_groups(E(48, dtype=torch.int8), 2, 3, 8, g, 2, scales=s))
    _bad(lambda: api.quantize_groups_batch([(src, 2, 3, 8, g, 2, E(2, device="meta"), None)]))
    _bad(lambda: api.softedge_encode(E(8, dtype=torch.float64), 1.0, 0.1, 5.0))
    _bad(lambda: api.softedge_decode(E(8, dtype=torch.int8), 1.0))
    _bad(lambda: api.group_absmax(src, 1, 6, 8, g, 3))
    _bad(lambda: api.cluster_by_absmax(E(4, dtype=torch.float16), 2))
    _bad(lambda: api.percentile_abs(E(4, dtype=torch.int8), [5.0]))


def test_noalloc_wrappers(rec):
    """The allocation-free calls check their tensors like the others and
    allocate nothing themselves (the recorder sees exactly one native call)."""
    src = E(100, dtype=torch.float16)
    out = E(2)
    assert api.percentile_abs_noalloc(src, [5.0, 99.9], out) is out
    _bad(lambda: api.percentile_abs_noalloc(src, [5.0, 99.9], E(3)))
    _bad(lambda: api.percentile_abs_noalloc(src, [5.0], E(1, dtype=torch.float16)))
    _bad(lambda: api.percentile_abs_noalloc(src, [5.0], E(1, device="meta")))
    _bad(lambda: api.percentile_abs_noalloc(E(100, dtype=torch.int32), [5.0], E(1)))
    thr = E(3)
    assert api.softedge_calibrate_noalloc(src, thr, alpha=0.1) is thr
    _bad(lambda: api.softedge_calibrate_noalloc(src, E(2)))
    _bad(lambda: api.softedge_calibrate_noalloc(src, E(3, device="meta")))
    assert rec.calls == ["ssmq_percentile_abs_noalloc", "ssmq_softedge_calibrate_noalloc"]


def test_scan_time_segments_and_carry_in_checks(rec):
    """Time segments: the workspace is sized by the library's query only for
    a split call and checked when supplied; dec_final and the carry-in's
    tensors are checked like every other tensor."""
    b, d, L, G, N = 2, 8, 64, 1, 16
    x, dt = E(b, d, L, dtype=torch.int8), E(b, d, L, dtype=torch.float16)
    Bq = E(b, G, N, L, dtype=torch.int8)
    args = (x, dt, E(d, N), Bq, Bq, E(4), E(4), 4)
    kw = dict(x_group=E(d, dtype=torch.int32), x_scale=E(2))
    api.selective_scan(*args, time_segments=2, **kw)
    api.selective_scan(*args, time_segments=2, workspace=E(512 + 255, dtype=torch.uint8), **kw)
    _bad(lambda: api.selective_scan(*args, time_segments=2,
                                    workspace=E(512, dtype=torch.uint8), **kw))
    _bad(lambda: api.selective_scan(*args, time_segments=2,
                                    workspace=E(1024, dtype=torch.int8), **kw))
    api.selective_scan(*args, dec_final=E(b, d, N), **kw)
    _bad(lambda: api.selective_scan(*args, dec_final=E(b, d), **kw))
    _bad(lambda: api.selective_scan(*args, dec_final=E(b, d, N, dtype=torch.float16), **kw))
    y = E(b, d, L, dtype=torch.float16)
    carry = lambda **k: api.selective_scan_carry_in(*args, k.pop("h", E(b, d, N)),
                                                    k.pop("y", y), **k)
    carry()
    carry(h_final=E(b, d, N), D=E(d), z=E(b, d, L, dtype=torch.float16), dt_bias=E(d))
    _bad(lambda: carry(h=E(b, d, N - 1)))
    _bad(lambda: carry(y=E(b, d, L)))
    _bad(lambda: carry(h_final=E(b, d)))
    _bad(lambda: carry(z=E(b, d, L - 1, dtype=torch.float16)))
    assert rec.calls.count("ssmq_selective_scan_carry_in") == 2
    assert rec.calls.count("ssmq_selective_scan_w8") == 3
