"""Seeded synthetic inputs shaped like the pages' workloads.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no quantization, no thresholds, no scan).  Both the CUDA
path and the CPU oracle consume exactly the arrays it returns.

Every tensor comes from ``numpy.random.default_rng(SeedSequence([seed, idx]))``
with ``idx`` the workload's index below, drawn in the order written in each
function.  Activations are binary16 (numpy float16), parameters float32.

Workloads (sizes from the pages' model families):
  0 tiny      Mamba-1 scan, b=1 L=256 d=64 N=16
  1 m130m     Mamba-130M-shaped layer scan, b=8 L=2048 d=1536 N=16, z gate,
              0.1% channel-persistent outlier channels x50
  2 ssd27b    Mamba-2-2.7B-shaped SSD scan, b=4 L=4096 H=80 P=64 N=128 G=1
  3 decode8b  Mamba-2-8B-shaped decode, b=64 H=128 P=64 N=128 G=8, fp32 state
  4 softedge  Mamba-130M layer with Student-t(3) x plus 0.05% outliers x100..1000,
              b=16 L=8192 d=1536 N=16
"""
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

F16_MAX = 65504.0


@dataclass
class Workload:
    name: str
    index: int
    kind: str  # "m1", "ssd", "decode"
    dims: dict = field(default_factory=dict)


WORKLOADS = {
    "tiny": Workload("tiny", 0, "m1", dict(batch=1, seqlen=256, dim=64, dstate=16, ngroups=1,
                                          state_group_size=16, x_clusters=1, gate=False)),
    "m130m": Workload("m130m", 1, "m1", dict(batch=8, seqlen=2048, dim=1536, dstate=16,
                                            ngroups=1, state_group_size=4, x_clusters=8,
                                            gate=True)),
    "ssd27b": Workload("ssd27b", 2, "ssd", dict(batch=4, seqlen=4096, nheads=80, headdim=64,
                                               dstate=128, ngroups=1, state_group_size=8,
                                               x_clusters=8, chunk=256, gate=False)),
    "decode8b": Workload("decode8b", 3, "decode", dict(batch=64, nheads=128, headdim=64,
                                                      dstate=128, ngroups=8, state_group_size=8,
                                                      x_clusters=8, steps=1000, gate=False)),
    "softedge": Workload("softedge", 4, "m1", dict(batch=16, seqlen=8192, dim=1536, dstate=16,
                                                  ngroups=1, state_group_size=4, x_clusters=1,
                                                  gate=True)),
}


def rng_for(index: int, seed: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, index]))


def _normal(rng, shape, mean=0.0, std=1.0):
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    if mean != 0.0:
        a += np.float32(mean)
    return a


def _f16(a):
    return np.clip(a, -F16_MAX, F16_MAX).astype(np.float16)


def a_log_uniform(rng, shape):
    """A = -exp(U(0, ln 16)), the Mamba real-diagonal initialisation range."""
    return (-np.exp(rng.uniform(0.0, np.log(16.0), size=shape))).astype(np.float32)


def m1_inputs(batch, seqlen, dim, dstate, ngroups=1, *, gate=True, seed=0, index=1,
              a_mode="log_uniform", outlier_frac=0.0, outlier_mul=50.0, x_dist="normal",
              spike_frac=0.0, spike_range=(100.0, 1000.0), with_bias=False, with_h0=False):
    """Raw fp activations for one Mamba-1 layer scan.

    Draw order: x, dt, z (if gate), B, C, A (if random), D, outlier channels
    or spike positions/factors, dt_bias (if requested), h0 (if requested).
    Layouts: x, dt, z (b, d, L); B, C (b, G, N, L); A (d, N).
    """
    rng = rng_for(index, seed)
    b, L, d, N, G = batch, seqlen, dim, dstate, ngroups
    if x_dist == "student_t3":
        x = rng.standard_t(3, size=(b, d, L)).astype(np.float32)
    else:
        x = _normal(rng, (b, d, L))
    dt = _normal(rng, (b, d, L), mean=-4.0, std=0.5)
    z = _normal(rng, (b, d, L)) if gate else None
    B = _normal(rng, (b, G, N, L))
    Cm = _normal(rng, (b, G, N, L))
    if a_mode == "s4d_real":
        A = np.broadcast_to(-(np.arange(N, dtype=np.float32) + 1.0), (d, N)).copy()
    else:
        A = a_log_uniform(rng, (d, N))
    D = _normal(rng, (d,))
    outlier_channels = spike_positions = None
    if outlier_frac > 0:
        n_out = int(round(outlier_frac * d))
        outlier_channels = np.sort(rng.choice(d, size=n_out, replace=False))
        x[:, outlier_channels, :] *= np.float32(outlier_mul)
    if spike_frac > 0:
        n_sp = int(round(spike_frac * x.size))
        pos = rng.choice(x.size, size=n_sp, replace=False)
        fac = rng.uniform(spike_range[0], spike_range[1], size=n_sp).astype(np.float32)
        flat = x.reshape(-1)
        flat[pos] *= fac
        spike_positions = np.sort(pos)
    dt_bias = _normal(rng, (d,), std=0.1) if with_bias else None
    h0 = _normal(rng, (b, d, N), std=0.1) if with_h0 else None
    return dict(x=_f16(x), dt=_f16(dt), z=None if z is None else _f16(z), B=_f16(B),
                C=_f16(Cm), A=A, D=D, dt_bias=dt_bias, h0=h0,
                outlier_channels=outlier_channels, spike_positions=spike_positions)


def ssd_inputs(batch, seqlen, nheads, headdim, dstate, ngroups=1, *, gate=False, seed=0,
               index=2, with_bias=False, with_h0=False, x_std=1.0):
    """Raw fp activations for one Mamba-2 SSD layer.

    Draw order: x, dt, z (if gate), B, C, A, D, dt_bias, h0.
    Layouts: x, z (b, L, H, P); dt (b, L, H); B, C (b, L, G, N); A, D (H,).
    """
    rng = rng_for(index, seed)
    b, L, H, P, N, G = batch, seqlen, nheads, headdim, dstate, ngroups
    x = _normal(rng, (b, L, H, P), std=x_std)
    dt = _normal(rng, (b, L, H), mean=-4.0, std=0.5)
    z = _normal(rng, (b, L, H, P)) if gate else None
    B = _normal(rng, (b, L, G, N))
    Cm = _normal(rng, (b, L, G, N))
    A = a_log_uniform(rng, (H,))
    D = _normal(rng, (H,))
    dt_bias = _normal(rng, (H,), std=0.1) if with_bias else None
    h0 = _normal(rng, (b, H, P, N), std=0.1) if with_h0 else None
    return dict(x=_f16(x), dt=_f16(dt), z=None if z is None else _f16(z), B=_f16(B),
                C=_f16(Cm), A=A, D=D, dt_bias=dt_bias, h0=h0)


def decode_inputs(batch, nheads, headdim, dstate, ngroups, steps, *, gate=False, seed=0,
                  index=3, state_std=0.1):
    """Raw inputs for a chain of single-token decode steps.

    Draw order: state, then per-step stacks x, dt, B, C, (z), then A, D.
    Layouts: state (b, H, P, N) float32; x (S, b, H, P); dt (S, b, H);
    B, C (S, b, G, N); A, D (H,).
    """
    rng = rng_for(index, seed)
    b, H, P, N, G, S = batch, nheads, headdim, dstate, ngroups, steps
    state = _normal(rng, (b, H, P, N), std=state_std)
    x = _normal(rng, (S, b, H, P))
    dt = _normal(rng, (S, b, H), mean=-4.0, std=0.5)
    B = _normal(rng, (S, b, G, N))
    Cm = _normal(rng, (S, b, G, N))
    z = _normal(rng, (S, b, H, P)) if gate else None
    A = a_log_uniform(rng, (H,))
    D = _normal(rng, (H,))
    return dict(state=state, x=_f16(x), dt=_f16(dt), B=_f16(B), C=_f16(Cm),
                z=None if z is None else _f16(z), A=A, D=D)


def workload_inputs(name: str, seed: int = 0, **overrides):
    """Raw inputs of one named workload at its full size (overrides shrink it)."""
    w = WORKLOADS[name]
    dm = dict(w.dims)
    dm.update(overrides)
    if w.kind == "m1":
        kw = dict(gate=dm["gate"], seed=seed, index=w.index)
        if name == "tiny":
            kw["a_mode"] = "s4d_real"
        if name == "m130m":
            kw.update(outlier_frac=0.001, outlier_mul=50.0)
        if name == "softedge":
            kw.update(x_dist="student_t3", spike_frac=0.0005)
        return dm, m1_inputs(dm["batch"], dm["seqlen"], dm["dim"], dm["dstate"], dm["ngroups"],
                             **kw)
    if w.kind == "ssd":
        return dm, ssd_inputs(dm["batch"], dm["seqlen"], dm["nheads"], dm["headdim"],
                              dm["dstate"], dm["ngroups"], gate=dm["gate"], seed=seed,
                              index=w.index)
    return dm, decode_inputs(dm["batch"], dm["nheads"], dm["headdim"], dm["dstate"],
                             dm["ngroups"], dm["steps"], gate=dm["gate"], seed=seed,
                             index=w.index)


def random_codes(rng: np.random.Generator, shape, lo=-127, hi=127):
    """Uniform random int8 codes (a synthetic already-quantized operand)."""
    return rng.integers(lo, hi + 1, size=shape, dtype=np.int64).astype(np.int8)


def random_scales(rng: np.random.Generator, n, lo=0.005, hi=0.05):
    """Positive fp32 scales drawn log-uniformly in [lo, hi]."""
    return np.exp(rng.uniform(np.log(lo), np.log(hi), size=n)).astype(np.float32)


def random_bytes(rng: np.random.Generator, shape):
    return rng.integers(0, 256, size=shape, dtype=np.int64).astype(np.uint8)
