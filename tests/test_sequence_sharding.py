"""Sequence sharding of the SSD scan (a slice per rank): the decomposition the
GPU path implements, pinned on the CPU against the oracle's unsplit scan, and
the summary exchange over gloo ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from problems import oracle_kwargs, ssd_problem


def _total_log2_decay(p, sl):
    """sum_t delta_t A_h log2(e) over the steps of slice sl, per (b, h)"""
    dt = p["dt"][:, sl].astype(np.float64)
    bias = 0.0 if p["dt_bias"] is None else p["dt_bias"].astype(np.float64)
    delta = np.logaddexp(0.0, dt + bias)
    return (delta * p["A"].astype(np.float64)).sum(axis=1) * np.log2(np.e)


def _fold(h_ends, decs):
    h = np.zeros_like(h_ends[0])
    for he, d in zip(h_ends, decs):
        h = np.exp2(d)[..., None, None] * h + he
    return h


def _slice(p, sl):
    q = dict(p)
    for k in ("x", "dt", "z", "B", "C"):
        if q[k] is not None:
            q[k] = np.ascontiguousarray(p[k][:, sl])
    return q


@pytest.mark.parametrize("cuts", [(0, 128, 300), (0, 77, 78, 200, 300)])
def test_slices_fold_to_the_unsplit_scan(orc, cuts):
    """Slices scanned from zero (the first from h0), folded with
    h <- exp2(dec) h + h_end, give the unsplit final state; each slice's y
    plus the y of its carried start state (the oracle's scan of the slice from
    that state minus its scan from zero) is the unsplit y."""
    b, L, H = 1, 300, 2
    p = ssd_problem(930, b, L, H, 64, 128, gate=True, h0=True, bias=True)
    yo, ho = orc.ssd_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["B_scale"], p["C_scale"],
                          8, **oracle_kwargs(p))
    bounds = list(cuts) + [L]
    h_ends, decs = [], []
    for r in range(len(bounds) - 1):
        sl = slice(bounds[r], bounds[r + 1])
        q = _slice(p, sl)
        if r > 0:
            q["h0"] = None
        kw = oracle_kwargs(q)
        y0, he = orc.ssd_scan(q["x"], q["dt"], q["A"], q["B"], q["C"], q["B_scale"],
                              q["C_scale"], 8, **kw)
        if r > 0:
            carry = _fold(h_ends, decs).reshape(b, H, 64, 128)
            kw["h0"] = carry.astype(np.float32).astype(np.float64)
            y1, _ = orc.ssd_scan(q["x"], q["dt"], q["A"], q["B"], q["C"], q["B_scale"],
                                 q["C_scale"], 8, **kw)
            kw["h0"] = np.zeros_like(kw["h0"])
            y0z, _ = orc.ssd_scan(q["x"], q["dt"], q["A"], q["B"], q["C"], q["B_scale"],
                                  q["C_scale"], 8, **kw)
            y0 = y0 + (y1 - y0z)
        np.testing.assert_allclose(y0, yo[:, sl], rtol=0, atol=2e-6 * np.abs(yo).max())
        h_ends.append(he.reshape(b, H, 64, 128))
        decs.append(_total_log2_decay(p, sl))
    hf = _fold(h_ends, decs).reshape(ho.shape)
    np.testing.assert_allclose(hf, ho, rtol=0, atol=1e-9 * np.abs(ho).max())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        from quantized_state_space_b200 import sharded
        g = torch.Generator().manual_seed(100 + rank)
        h_end = torch.randn(2, 3, 4, 5, generator=g)
        dec = -torch.rand(2, 3, generator=g)
        hs, ds = sharded.exchange(h_end, dec)
        out[rank] = ([h.numpy() for h in hs], [d.numpy() for d in ds], h_end.numpy(),
                     dec.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_exchange_over_three_gloo_ranks():
    """Every rank receives every rank's summary, in rank order."""
    world = 3
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    for r in range(world):
        hs, ds, _, _ = res[r]
        for q in range(world):
            np.testing.assert_array_equal(hs[q], res[q][2])
            np.testing.assert_array_equal(ds[q], res[q][3])


def test_sharded_call_rejects_unshared_arguments():
    """Only the arguments that both the slice scan and its carry-in take are
    accepted (an int8-y request, for one, has no carry-in form)."""
    from quantized_state_space_b200 import sharded
    with pytest.raises(TypeError, match="y_group"):
        sharded.ssd_chunk_scan_sequence_sharded(None, None, None, None, None, None, None, 8,
                                                y_group=None)


def test_m1_sharded_call_rejects_unshared_arguments():
    """The Mamba-1 slice call takes the scan's x / gate / delta arguments; an
    int8-y request or a time split has no sharded form."""
    from quantized_state_space_b200 import sharded
    for bad in ("y_group", "time_segments"):
        with pytest.raises(TypeError, match=bad):
            sharded.selective_scan_sequence_sharded(None, None, None, None, None, None, None, 4,
                                                    **{bad: None})


def _m1_fold(h_ends, decs):
    h = np.zeros_like(h_ends[0])
    for he, d in zip(h_ends, decs):
        h = np.exp2(d) * h + he
    return h


@pytest.mark.parametrize("cuts", [(0, 100, 250), (0, 1, 2, 180)])
def test_m1_slices_fold_to_the_unsplit_scan(orc, cuts):
    """Mamba-1: slices scanned from zero (the first from h0), folded with
    h <- exp2(dec) h + h_end, dec = A_cn log2(e) sum_t delta_t per (b, c, n),
    give the unsplit final state; each slice's y plus the y of its carried
    start state is the unsplit y."""
    from problems import m1_problem
    b, L, d, N_ = 2, 300, 16, 8
    p = m1_problem(935, b, L, d, N_, gate=True, h0=True, bias=True)
    sc = lambda q, **kw: orc.m1_scan(q["x"], q["dt"], q["A"], q["B"], q["C"], q["B_scale"],
                                     q["C_scale"], q["state_group_size"], **kw)
    yo, ho = sc(p, **oracle_kwargs(p))
    bounds = list(cuts) + [L]
    h_ends, decs = [], []
    for r in range(len(bounds) - 1):
        sl = slice(bounds[r], bounds[r + 1])
        q = dict(p)
        for k in ("x", "dt", "z", "B", "C"):
            q[k] = np.ascontiguousarray(p[k][..., sl])
        if r > 0:
            q["h0"] = None
        kw = oracle_kwargs(q)
        y0, he = sc(q, **kw)
        if r > 0:
            carry = _m1_fold(h_ends, decs)
            kw["h0"] = carry.astype(np.float32).astype(np.float64)
            y1, _ = sc(q, **kw)
            kw["h0"] = np.zeros_like(kw["h0"])
            y0z, _ = sc(q, **kw)
            y0 = y0 + (y1 - y0z)
        np.testing.assert_allclose(y0.reshape(b, d, -1), yo.reshape(b, d, L)[..., sl], rtol=0,
                                   atol=2e-6 * np.abs(yo).max())
        h_ends.append(he.reshape(b, d, N_))
        dv = q["dt"].astype(np.float64) + p["dt_bias"].astype(np.float64)[None, :, None]
        decs.append(np.logaddexp(0.0, dv).sum(axis=2)[:, :, None]
                    * p["A"].astype(np.float64)[None] * np.log2(np.e))
    hf = _m1_fold(h_ends, decs)
    np.testing.assert_allclose(hf, ho.reshape(hf.shape), rtol=0, atol=1e-9 * np.abs(ho).max())


class _OracleKernels:
    """Stand-ins for the library calls of the Mamba-1 sharded path, computed
    by the oracle in float64 on the host (the orchestration under test is the
    rank logic: who starts from h0, which summaries are folded, where the
    carry-in goes)."""

    def __init__(self, O, gs, kw):
        self.O, self.gs, self.kw = O, gs, kw

    def _scan(self, x, dt, A, B, C, Bs, Cs, h0):
        kw = dict(self.kw)
        kw["h0"] = None if h0 is None else h0.numpy().astype(np.float64)
        y, h = self.O.m1_scan(x.numpy(), dt.numpy(), A.numpy(), B.numpy(), C.numpy(),
                              Bs.numpy(), Cs.numpy(), self.gs, **kw)
        b, d, L = x.shape
        return torch.from_numpy(y.reshape(b, d, L)), torch.from_numpy(h.reshape(b, d, -1))

    def selective_scan(self, x, dt, A, B, C, Bs, Cs, gs, h0=None, dec_final=None, **_):
        y, h = self._scan(x, dt, A, B, C, Bs, Cs, h0)
        dv = dt.numpy().astype(np.float64) + self.kw["dt_bias"][None, :, None]
        dec = (np.logaddexp(0.0, dv).sum(axis=2)[:, :, None] * A.numpy().astype(np.float64)[None]
               * np.log2(np.e))
        dec_final.copy_(torch.from_numpy(dec))
        return y, h

    @staticmethod
    def state_chain(hs, ds):
        h = torch.zeros_like(hs[0])
        for he, d in zip(hs, ds):
            h = torch.exp2(d) * h + he
        return h

    def selective_scan_carry_in(self, x, dt, A, B, C, Bs, Cs, gs, h_carry, y, **_):
        y1, _ = self._scan(x, dt, A, B, C, Bs, Cs, h_carry)
        y0, _ = self._scan(x, dt, A, B, C, Bs, Cs, None)
        y += y1 - y0


def _m1_sharded_worker(rank, world, port, out, cuts):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        from oracle import oracle as O
        from problems import m1_problem
        from quantized_state_space_b200 import sharded
        p = m1_problem(960, 2, 200, 8, 8, gate=True, h0=True, bias=True)
        kw = dict(D=p["D"], z=None, dt_bias=p["dt_bias"], x_group=p["x_group"],
                  x_scale=p["x_scale"])
        sl = slice(cuts[rank], cuts[rank + 1])
        q = {k: (np.ascontiguousarray(p[k][..., sl]) if k in ("x", "dt", "z", "B", "C") else p[k])
             for k in p}
        kw["z"] = q["z"].astype(np.float64)
        sharded.api = _OracleKernels(O, p["state_group_size"], kw)
        T = lambda a: torch.from_numpy(np.ascontiguousarray(a))
        y, hf = sharded.selective_scan_sequence_sharded(
            T(q["x"]), T(q["dt"]), T(q["A"]), T(q["B"]), T(q["C"]), T(q["B_scale"]),
            T(q["C_scale"]), p["state_group_size"], h0=T(p["h0"]))
        out[rank] = (y.numpy(), hf.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts", [(0, 90, 200), (0, 50, 51, 200)])
def test_m1_sharded_orchestration_over_gloo_ranks(orc, cuts):
    """The Mamba-1 sequence-sharded call on 2 and 3 gloo ranks, the library
    calls stood in for by the oracle: the slices' y concatenated and every
    rank's final state against the oracle's unsplit scan."""
    world = len(cuts) - 1
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_m1_sharded_worker, args=(world, port, out, cuts), nprocs=world,
                           join=True, start_method="spawn")
        res = dict(out)
    from problems import m1_problem
    p = m1_problem(960, 2, 200, 8, 8, gate=True, h0=True, bias=True)
    kw = oracle_kwargs(p)
    yo, ho = orc.m1_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["B_scale"], p["C_scale"],
                         p["state_group_size"], **kw)
    # the exchanged log2 decays are fp32 (as the library's): 1e-6 of the
    # largest value; a wrong start state or fold order is off by O(1)
    y = np.concatenate([res[r][0] for r in range(world)], axis=-1)
    np.testing.assert_allclose(y, yo.reshape(y.shape), rtol=0, atol=1e-6 * np.abs(yo).max())
    for r in range(world):
        np.testing.assert_allclose(res[r][1], ho.reshape(res[r][1].shape), rtol=0,
                                   atol=1e-6 * np.abs(ho).max())


class _OracleSsdKernels:
    """The SSD sharded path's library calls, stood in for by the oracle."""

    def __init__(self, O, gs, kw):
        self.O, self.gs, self.kw = O, gs, kw

    def _scan(self, x, dt, A, B, C, Bs, Cs, h0):
        kw = dict(self.kw)
        kw["h0"] = None if h0 is None else h0.numpy().astype(np.float64)
        y, h = self.O.ssd_scan(x.numpy(), dt.numpy(), A.numpy(), B.numpy(), C.numpy(),
                               Bs.numpy(), Cs.numpy(), self.gs, **kw)
        b, L, H, P = x.shape  # the oracle's y is (b H, L, P)
        y = np.ascontiguousarray(y.reshape(b, H, L, P).transpose(0, 2, 1, 3))
        return torch.from_numpy(y), torch.from_numpy(h.reshape(b, H, P, -1))

    def ssd_chunk_scan(self, x, dt, A, B, C, Bs, Cs, gs, h0=None, dec_final=None, **_):
        y, h = self._scan(x, dt, A, B, C, Bs, Cs, h0)
        dv = dt.numpy().astype(np.float64) + self.kw["dt_bias"][None, None, :]
        dec = np.logaddexp(0.0, dv).sum(axis=1) * A.numpy().astype(np.float64) * np.log2(np.e)
        dec_final.copy_(torch.from_numpy(dec))
        return y, h

    state_chain = staticmethod(lambda hs, ds: _fold_t(hs, ds))

    def ssd_carry_in(self, x, dt, A, B, C, Bs, Cs, gs, h_carry, y, **_):
        y1, _ = self._scan(x, dt, A, B, C, Bs, Cs, h_carry)
        y0, _ = self._scan(x, dt, A, B, C, Bs, Cs, None)
        y += y1 - y0


def _fold_t(hs, ds):
    h = torch.zeros_like(hs[0])
    for he, d in zip(hs, ds):
        h = torch.exp2(d).reshape(d.shape + (1,) * (he.dim() - d.dim())) * h + he
    return h


def _ssd_sharded_worker(rank, world, port, out, cuts):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        from oracle import oracle as O
        from quantized_state_space_b200 import sharded
        p = ssd_problem(965, 1, 300, 2, 64, 128, gate=False, h0=True, bias=True)
        kw = oracle_kwargs(p)
        kw.pop("h0")
        sl = slice(cuts[rank], cuts[rank + 1])
        q = {k: (np.ascontiguousarray(p[k][:, sl]) if k in ("x", "dt", "B", "C") else p[k])
             for k in p}
        sharded.api = _OracleSsdKernels(O, 8, kw)
        T = lambda a: torch.from_numpy(np.ascontiguousarray(a))
        y, hf = sharded.ssd_chunk_scan_sequence_sharded(
            T(q["x"]), T(q["dt"]), T(q["A"]), T(q["B"]), T(q["C"]), T(q["B_scale"]),
            T(q["C_scale"]), 8, h0=T(p["h0"]))
        out[rank] = (y.numpy(), hf.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_ssd_sharded_orchestration_over_gloo_ranks(orc):
    """The SSD sequence-sharded call on 3 gloo ranks, the library calls stood
    in for by the oracle, against the oracle's unsplit scan."""
    cuts = (0, 77, 201, 300)
    world = len(cuts) - 1
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_ssd_sharded_worker, args=(world, port, out, cuts), nprocs=world,
                           join=True, start_method="spawn")
        res = dict(out)
    p = ssd_problem(965, 1, 300, 2, 64, 128, gate=False, h0=True, bias=True)
    yo, ho = orc.ssd_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["B_scale"], p["C_scale"],
                          8, **oracle_kwargs(p))
    y = np.concatenate([res[r][0] for r in range(world)], axis=1)
    yo = yo.reshape(1, 2, 300, 64).transpose(0, 2, 1, 3)  # (b H, L, P) -> (b, L, H, P)
    np.testing.assert_allclose(y, yo, rtol=0, atol=1e-6 * np.abs(yo).max())
    for r in range(world):
        np.testing.assert_allclose(res[r][1], ho.reshape(res[r][1].shape), rtol=0,
                                   atol=1e-6 * np.abs(ho).max())
