"""GPU quantizers vs the oracle, bit for bit (Quamba-SE write-up sections 1,
2.1, 2.2; Quamba2 abstract)."""
import numpy as np
import pytest
import torch

from gpu_util import H, T, dev, status_word
from quantized_state_space_b200 import _native as N
from quantized_state_space_b200 import api, calibrate, synth

pytestmark = pytest.mark.gpu

SHAPES = [  # (outer, mid, inner): row path, column path, general path, ragged tails
    (3, 5, 2048), (2, 37, 1003), (777, 80, 1), (5, 17, 1), (1, 1, 7), (4, 48, 16),
    (9, 1536, 3), (1, 3, 100_001),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dtype", [np.float16, np.float32])
def test_quantize_static(orc, shape, dtype):
    outer, mid, inner = shape
    rng = np.random.default_rng(sum(shape))
    k = min(6, mid)
    gmap = rng.integers(0, k, size=mid).astype(np.int32)
    x = (rng.standard_normal(shape) * rng.choice([0.1, 1, 20], size=shape)).astype(dtype)
    sc = synth.random_scales(rng, k, 0.01, 0.2)
    qg, _ = api.quantize_groups(T(x), outer, mid, inner, T(gmap), k, scales=T(sc))
    qo, _, _ = orc.quantize_groups(x, outer, mid, inner, gmap, k, orc.SCALE_STATIC, sc)
    np.testing.assert_array_equal(H(qg), qo)


@pytest.mark.parametrize("shape", SHAPES)
def test_quantize_absmax(orc, shape):
    outer, mid, inner = shape
    rng = np.random.default_rng(7 + sum(shape))
    k = min(5, mid)
    gmap = rng.integers(0, k, size=mid).astype(np.int32)
    x = (rng.standard_normal(shape) * 3).astype(np.float16)
    qg, sg = api.quantize_groups(T(x), outer, mid, inner, T(gmap), k, absmax=True)
    qo, so, _ = orc.quantize_groups(x, outer, mid, inner, gmap, k, orc.SCALE_ABSMAX)
    np.testing.assert_array_equal(H(sg), so)
    np.testing.assert_array_equal(H(qg), qo)


@pytest.mark.parametrize("dtype", [np.float16, np.float32])
def test_quantize_column_groups_of_8(orc, dtype):
    """Column path with 8-column groups (Mamba-2 B/C: one scale per 8
    states) and a map whose 8-column blocks are partly mixed: each half of a
    16-element vector takes its own scale, mixed blocks go element by element."""
    rng = np.random.default_rng(88)
    outer, mid = 300, 128
    for gmap in (np.arange(mid, dtype=np.int32) // 8,
                 np.where(np.arange(mid) % 24 < 20, np.arange(mid) // 8, 3).astype(np.int32)):
        k = int(gmap.max()) + 1
        x = (rng.standard_normal((outer, mid)) * 4).astype(dtype)
        sc = synth.random_scales(rng, k, 0.01, 0.2)
        qg, _ = api.quantize_groups(T(x), outer, mid, 1, T(gmap), k, scales=T(sc))
        qo, _, _ = orc.quantize_groups(x, outer, mid, 1, gmap, k, orc.SCALE_STATIC, sc)
        np.testing.assert_array_equal(H(qg), qo)


def test_quantize_all_f16_patterns(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = bits.view(np.float16).copy()
    for s in (1.0, 0.0078125, 3.3e-5, 517.0):
        st = status_word()
        qg, _ = api.quantize_groups(T(x), 1, 1, x.size, T(np.zeros(1, np.int32)), 1,
                                    scales=T(np.array([s], np.float32)), status=st)
        qo, _, nf = orc.quantize_groups(x, 1, 1, x.size, [0], 1, orc.SCALE_STATIC,
                                        np.array([s], np.float32))
        np.testing.assert_array_equal(H(qg), qo)
        assert nf > 0 and int(H(st)[0]) & N.DEV_NONFINITE


def test_quantize_all_f32_patterns(orc):
    """Every binary32 bit pattern (2^32, in 16 slices of 2^28) at one scale
    whose reciprocal is inexact: the codes equal the oracle's byte for byte,
    including every near-tie quotient, the clamp and the non-finite inputs."""
    s = np.array([0.7310586], np.float32)
    n = 1 << 28
    base = np.arange(n, dtype=np.uint32)
    bits = np.empty(n, np.uint32)
    sc, g0 = T(s), T(np.zeros(1, np.int32))
    xg = torch.empty(n, dtype=torch.float32, device="cuda")
    for k in range(16):
        np.add(base, np.uint32(k * n), out=bits)
        x = bits.view(np.float32)
        xg.copy_(torch.from_numpy(x))
        qg, _ = api.quantize_groups(xg, 1, 1, n, g0, 1, scales=sc)
        qo, _, _ = orc.quantize_groups(x, 1, 1, n, [0], 1, orc.SCALE_STATIC, s)
        got = H(qg)
        if not np.array_equal(got, qo):
            i = int(np.flatnonzero(got != qo)[0])
            raise AssertionError("pattern 0x%08x: gpu %d oracle %d" % (int(bits[i]), got[i], qo[i]))


def test_quantize_status_bits():
    x = T(np.ones(64, np.float16))
    st = status_word()
    api.quantize_groups(x, 1, 64, 1, T(np.full(64, 3, np.int32)), 2, scales=T(np.ones(2, np.float32)),
                        status=st)
    torch.cuda.synchronize()
    assert int(H(st)[0]) & N.DEV_BAD_GROUP
    st.zero_()
    q, _ = api.quantize_groups(x, 1, 64, 1, T(np.zeros(64, np.int32)), 1,
                               scales=T(np.array([-1.0], np.float32)), status=st)
    assert int(H(st)[0]) & N.DEV_BAD_SCALE and not H(q).any()


def test_pipeline_wait_gives_up(orc, monkeypatch):
    """Failure detection on the GPU without a fault: with SSMQ_WAIT_LIMIT=0
    every wait of the quantizer's bulk-copy pipeline gives up at once.  The
    kernel must still return (after draining the copies it issued), the call
    reports SSMQ_DEV_TIMEOUT in the status word, and the context stays usable:
    the next call, with the normal limit, gives the oracle's codes."""
    rng = np.random.default_rng(11)
    b, d, L = 4, 96, 4096  # many tiles per CTA
    x = rng.standard_normal((b, d, L)).astype(np.float16)
    grp = rng.integers(0, 4, size=d).astype(np.int32)
    sc = synth.random_scales(rng, 4, 0.01, 0.05)
    xt, gt, st_ = T(x), T(grp), T(sc)
    st = status_word()
    monkeypatch.setenv("SSMQ_WAIT_LIMIT", "0")
    api.quantize_groups(xt, b, d, L, gt, 4, scales=st_, status=st)
    torch.cuda.synchronize()
    assert int(H(st)[0]) & N.DEV_TIMEOUT
    monkeypatch.delenv("SSMQ_WAIT_LIMIT")
    st.zero_()
    q, _ = api.quantize_groups(xt, b, d, L, gt, 4, scales=st_, status=st)
    torch.cuda.synchronize()
    assert int(H(st)[0]) == 0
    qo, _, _ = orc.quantize_groups(x, b, d, L, grp, 4, orc.SCALE_STATIC, sc)
    np.testing.assert_array_equal(H(q), qo)


def test_quantize_m130m_x_full_size(orc):
    """Full-size Mamba-130M-shaped x with its sort-and-cluster scales."""
    _, raw = synth.workload_inputs("m130m")
    x = raw["x"]
    b, d, L = x.shape
    grp, sc = calibrate.m1_x_clusters(x, 8)
    og, osc = orc.cluster_by_absmax(orc.absmax_per_mid(x, b, d, L), 8)
    np.testing.assert_array_equal(grp, og)
    np.testing.assert_array_equal(sc, osc)
    qg, _ = api.quantize_groups(T(x), b, d, L, T(grp), 8, scales=T(sc))
    qo, _, _ = orc.quantize_groups(x, b, d, L, og, 8, orc.SCALE_STATIC, osc)
    np.testing.assert_array_equal(H(qg), qo)


def _batch_job(rng, shape, dtype, k):
    outer, mid, inner = shape
    k = min(k, mid)
    gmap = rng.integers(0, k, size=mid).astype(np.int32)
    x = (rng.standard_normal(shape) * rng.choice([0.1, 1, 20], size=shape)).astype(dtype)
    return x, gmap, k, synth.random_scales(rng, k, 0.01, 0.2)


def test_quantize_batch_vs_oracle_and_single_calls(orc):
    """One batch of eight jobs (row, column and general paths, binary16 and
    fp32, ragged, tiny and empty tensors) gives the oracle's codes and the
    same bytes as one call per job."""
    rng = np.random.default_rng(4242)
    specs = [((8, 1536, 256), np.float16), ((8, 16, 256), np.float16),
             ((8, 16, 256), np.float16), ((777, 80, 1), np.float32), ((2, 37, 1003), np.float16),
             ((1, 1, 7), np.float16), ((0, 5, 16), np.float16), ((3, 5, 2048), np.float32)]
    jobs, data = [], []
    for shape, dt in specs:
        x, gmap, k, sc = _batch_job(rng, shape, dt, 8)
        data.append((x, gmap, k, sc))
        jobs.append((T(x), *shape, T(gmap), k, T(sc), None))
    st = status_word()
    outs = api.quantize_groups_batch(jobs, status=st)
    assert int(H(st)[0]) == 0
    for (x, gmap, k, sc), q, (shape, _) in zip(data, outs, specs):
        qo, _, _ = orc.quantize_groups(x, *shape, gmap, k, orc.SCALE_STATIC, sc)
        np.testing.assert_array_equal(H(q), qo.reshape(shape))
        single, _ = api.quantize_groups(T(x), *shape, T(gmap), k, scales=T(sc))
        np.testing.assert_array_equal(H(q), H(single))


def test_quantize_batch_status_and_validation():
    x = T(np.ones(64, np.float16))
    st = status_word()
    api.quantize_groups_batch([(x, 1, 64, 1, T(np.full(64, 3, np.int32)), 2,
                                T(np.ones(2, np.float32)), None)], status=st)
    torch.cuda.synchronize()
    assert int(H(st)[0]) & N.DEV_BAD_GROUP
    with pytest.raises(N.SSMQError):
        api.quantize_groups_batch([(x, 1, 64, 1, T(np.zeros(64, np.int32)), 1,
                                    T(np.ones(1, np.float32)), None)] * 9)


# ---- soft-edge ---------------------------------------------------------------

@pytest.mark.parametrize("s,lo,hi,r", [(0.05, 0.1, 3.0, 2), (1.0 / 63, 0.02, 1.0, 2),
                                       (0.2, 0.0, 12.0, 2), (0.05, 0.1, 3.0, 1),
                                       (1.0, 1.0, 63.0, 2), (3e-6, 1e-5, 2e-4, 2)])
def test_softedge_encode_all_f16(orc, s, lo, hi, r):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = bits.view(np.float16).copy()
    s, lo, hi = np.float32(s), np.float32(lo), np.float32(hi)
    st = status_word()
    cg = api.softedge_encode(T(x), s, lo, hi, r, status=st)
    co, nf = orc.softedge_encode(x, s, lo, hi, r)
    np.testing.assert_array_equal(H(cg), co)
    assert int(H(st)[0]) & N.DEV_NONFINITE


def test_softedge_encode_f32_random(orc):
    rng = np.random.default_rng(3)
    x = (rng.standard_t(3, size=1_000_003) * 0.7).astype(np.float32)
    s, lo, hi = np.float32(0.031), np.float32(0.04), np.float32(2.9)
    np.testing.assert_array_equal(H(api.softedge_encode(T(x), s, lo, hi, 2)),
                                  orc.softedge_encode(x, s, lo, hi, 2)[0])


@pytest.mark.parametrize("s,r", [(1.0, 2), (0.0173, 2), (0.0173, 1), (2.5e-39, 2)])
def test_softedge_decode_all_codes(orc, s, r):
    codes = np.tile(np.arange(256, dtype=np.uint16).astype(np.uint8), 37)[:9001]
    dg = H(api.softedge_decode(T(codes), s, r))
    do = orc.softedge_decode(codes, np.float32(s), r)
    np.testing.assert_array_equal(dg.view(np.uint32), do.view(np.uint32))


def test_softedge_full_size_workload(orc):
    """Full-size soft-edge workload x (16 x 1536 x 8192), thresholds from the
    5th / 99.9th percentiles of |x|."""
    _, raw = synth.workload_inputs("softedge")
    x = raw["x"]
    s, lo, hi = calibrate.softedge_params(x)
    assert lo == np.float32(orc.percentile_abs(x, 5.0))
    assert hi == np.float32(orc.percentile_abs(x, 99.9))
    cg = H(api.softedge_encode(T(x), s, lo, hi, 2))
    co, _ = orc.softedge_encode(x, s, lo, hi, 2)
    np.testing.assert_array_equal(cg, co)
    # the page's "about 95% standard" holds by construction of L and H
    frac_std = float(np.mean((co >> 7) == 0))
    assert 0.93 < frac_std < 0.96
